"""fb_step (gates + out-of-block pass + in-block pass + merge) against the oracle
applying the same reuse policy, step by step (needs a B200).

Decisions are compared bit for bit; A_full within max-abs 2e-2 and mean-abs 1e-3,
L_full within 1e-3 (bf16 inputs, fp32 accumulation)."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu, torch_and_binding
from oracle import policy

pytestmark = pytest.mark.gpu


def _compare(w, flags=None, out_splits=0, sample=None, head_reuse_in=None):
    gpu, cache = run_policy_gpu(w, flags=flags, out_splits=out_splits, head_reuse_in=head_reuse_in)
    ref = policy.run_policy(w, flags=flags, sample=sample, head_reuse_in=head_reuse_in)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"{w.name} step {s}: decisions differ"
        if r.cos is not None and w.flags & W.GATE_HEAD:
            assert np.all(np.abs(r.cos - w.gamma) > 1e-5), "a similarity sits within rounding of gamma"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"{w.name} step {s}")
    return gpu, ref


def test_tiny():
    gpu, ref = _compare(W.tiny())
    assert ref[0].recompute.all() and not any(r.recompute.any() for r in ref[1:])


def test_tiny_sharp_forced_arms():
    w = W.tiny(sharp=32.0)
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w, flags=W.FORCE_REUSE)


def test_tiny_multi_split():
    _compare(W.tiny(), out_splits=3)


def test_locking_monotone_gqa():
    _compare(W.locking_tiny())


def test_caller_head_mask():
    w = W.locking_tiny(steps=3)
    rng = np.random.default_rng(0)
    masks = [None] + [rng.integers(0, 2, size=(w.problem.num_seqs, w.problem.num_heads_q)).astype(bool)
                      for _ in range(2)]
    _compare(w, head_reuse_in=masks)


def test_dllm_layer_full_size():
    """The 8B-dLLM layer workload at its full size, every row, all 32 steps."""
    gpu, ref = _compare(W.dllm_layer())
    dec = [bool(r.recompute.any()) for r in ref]
    assert dec[0] and any(dec[1:]) and not all(dec[1:])


def test_varlen_branches_full_size():
    gpu, ref = _compare(W.varlen_branches())
    per_branch = np.array([r.recompute[:, 0] for r in ref[1:]])
    assert per_branch.any() and not per_branch.all()   # branches decide differently


def test_long_context_gqa_reduced_both_arms():
    w = W.long_context_gqa(steps=3, prefix=2048 + 37)
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w, flags=W.FORCE_REUSE)


def test_video_reduced_gamma_gate():
    w = W.video(steps=4, block=256, prefix_blocks=2, heads=8)
    gpu, ref = _compare(w)
    assert any(r.recompute.any() and not r.recompute.all() for r in ref[1:])


def _threads(w):
    _, B = torch_and_binding()
    return B.plan_query(B.DeviceProblem(w.problem, "cpu"))


def _rows_vanish_workload(hq, hkv, blocks, prefix, flags, gamma, tau, seed=11):
    """Two steps with every block row active, then two in which every row is locked
    (the call has no query row at all): the gates still decide every head and the
    cache state still moves.  The queries never change, so a head's cosine is 1
    while it has rows."""
    rng = np.random.default_rng(seed)
    d = 128
    p_all = W.make_problem([np.arange(B) for B in blocks], [prefix] * len(blocks), blocks, hq, hkv, d)
    p_none = W.make_problem([np.zeros(0, np.int64) for _ in blocks], [prefix] * len(blocks), blocks, hq, hkv, d)
    k_out = W.normal_bf16(rng, (p_all.total_kv_out, hkv, d))
    v_out = W.normal_bf16(rng, (p_all.total_kv_out, hkv, d))
    q_blk = W.normal_bf16(rng, (p_all.total_kv_in, hq, d))
    k_blk = W.normal_bf16(rng, (p_all.total_kv_in, hkv, d))
    v_blk = W.normal_bf16(rng, (p_all.total_kv_in, hkv, d))
    n = np.ones(len(blocks), np.int32)
    steps = [W.StepInput(q=q_blk.copy(), k_in=k_blk, v_in=v_blk, n_updated=n.copy(), problem=p_all)
             for _ in range(2)]
    steps += [W.StepInput(q=q_blk[:0].copy(), k_in=k_blk, v_in=v_blk, n_updated=n.copy(), problem=p_none)
              for _ in range(2)]
    return W.Workload("rows_vanish", p_all, k_out, v_out, steps, tau=tau, gamma=gamma, flags=flags)


@pytest.mark.parametrize("flags", [W.GATE_HEAD, W.GATE_TAU, W.GATE_TAU_CUM, W.FORCE_REUSE, W.GATE_TAU | W.GATE_HEAD],
                         ids=["gamma", "tau", "tau_cum", "force_reuse", "tau_and_gamma"])
@pytest.mark.parametrize("hq,hkv,blocks", [(4, 4, (48, 29)), (8, 2, (32, 64))], ids=["warp_mma", "tensor_core"])
def test_calls_with_no_active_rows(flags, hq, hkv, blocks):
    """Degenerate calls (every row of every sequence locked) after calls with rows:
    decisions, validity and the cumulative counts match the oracle.  With no rows a
    head's cosine is 0 (a zero denominator), so the gamma gate recomputes; the score
    is computed for the call, never left over from the previous one."""
    w = _rows_vanish_workload(hq, hkv, list(blocks), 150, flags, gamma=0.5, tau=3)
    gpu, cache = run_policy_gpu(w)
    ocache = policy.OracleCache.empty(w.problem)
    ref = policy.run_policy(w, cache=ocache)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}: decisions differ"
        if r.a_full.shape[0]:
            assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"step {s}")
    S = w.problem.num_seqs
    assert np.array_equal(cache.valid.cpu().numpy()[:S].astype(bool), ocache.valid)
    assert np.array_equal(cache.m_acc.cpu().numpy()[:S], ocache.m_acc)
    if flags & W.GATE_HEAD:
        assert not ref[1].recompute.any() and ref[2].recompute.all()


@pytest.mark.parametrize("arm", ["tau", "gamma", "recompute", "reuse"])
def test_two_tile_sequences_with_one_and_no_rows(arm):
    """Two-tile kernel (one q-head per kv-head, a 300-row sequence) in a call that
    also holds a sequence with a single active row and one whose rows are all
    locked: work items with one row and an empty second tile, and items with no row
    at all; under the similarity gate the heads decide differently per sequence and
    the work-order pass puts the recomputing items first."""
    import dataclasses
    from test_gpu_reuse import _workload
    w = _workload([300, 40, 24], [np.arange(300), np.array([7]), np.zeros(0, np.int64)], 200, 2, 2, 128, steps=4)
    assert _threads(w)["kernel_name"] == "tc2_attn_kernel"
    flags = {"tau": None, "gamma": None, "recompute": W.FORCE_RECOMPUTE, "reuse": W.FORCE_REUSE}[arm]
    if arm == "gamma":
        w = dataclasses.replace(w, gamma=0.5, flags=W.GATE_HEAD | W.GATE_TAU)
    _, ref = _compare(w, flags=flags)
    if arm == "gamma":
        assert all(not r.recompute[0].any() and r.recompute[1:].all() for r in ref[1:])


@pytest.mark.parametrize("make", [
    lambda: W.dllm_layer(steps=4, prefix=2000, heads=8),
    lambda: W.dllm_layer(steps=4, prefix=2000, heads=8, head_dim=64),
    lambda: W.long_context_gqa(steps=3, batch=1, prefix=2085),
], ids=["warp_mma_d128", "warp_mma_d64", "tensor_core"])
def test_eight_cta_clusters(make):
    """Few groups on a long prefix: the plan splits every group's prefix over the
    largest portable cluster (8 CTAs), so the log-space combine reads seven remote
    partials through distributed shared memory; ragged last chunks; the forced
    recompute arm and the workload's own gates (reuse steps on the lean path)."""
    w = make()
    assert _threads(w)["splits"] == 8
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w)


def test_tensor_core_two_threads_per_row_varlen():
    """Grids of more than one wave run the tensor-core kernel with two softmax threads
    per row (the halves of a row swap their maxima every chunk): ragged varlen
    branches (prefix 300 + 37, chunks ending mid-way in both halves of a row), both
    forced arms and the gate."""
    w = W.varlen_branches(steps=4, prefix=337)
    plan = _threads(w)
    assert plan["kernel_name"] == "tc_attn_kernel" and plan["ctas"] > plan["num_sms"] and plan["threads"] == 320
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w, flags=W.FORCE_REUSE)
    _compare(w)


def test_tensor_core_two_threads_per_row_gqa_locking():
    """The same on a GQA batch of 40 sequences (320 groups, g = 4, half the block's
    rows locked), whose reuse steps take the lean path with its loads after the
    decision (the grid is more than one wave)."""
    w = W.long_context_gqa(steps=3, batch=40, prefix=203)
    plan = _threads(w)
    assert plan["threads"] == 320 and plan["lean_reuse"] == 1 and plan["lean_early"] == 0
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w, flags=W.FORCE_REUSE)


def test_determinism():
    w = W.varlen_branches(steps=3, prefix=512)
    a, _ = run_policy_gpu(w)
    b, _ = run_policy_gpu(w)
    for x, y in zip(a, b):
        assert np.array_equal(x["a_full"], y["a_full"]) and np.array_equal(x["l_full"], y["l_full"])


def test_two_tile_mha_ragged():
    """Two-tile tensor-core path: 300-token block (a full 256-row pair, then 44
    rows), prefix of 300 keys (ragged chunks in both segments), gamma gate."""
    w = W.video(steps=3, block=300, prefix_blocks=1, heads=4)
    _compare(w)
    _compare(w, flags=W.FORCE_REUSE)


def test_two_tile_mha_locking():
    """Two-tile path with SureLock-style locked rows (q_rows not the identity),
    two sequences deciding differently under the tau gate."""
    w = W.locking_tiny(steps=4, block=300, prefix=200, heads_q=2, heads_kv=2, head_dim=128, redraws=(3, 5))
    gpu, ref = _compare(w)
    for r in ref[1:]:   # tau = 4: sequence 0 (3 redraws) reuses, sequence 1 (5 redraws) recomputes
        assert not r.recompute[0].any() and r.recompute[1].all(), r.recompute


def test_cumulative_tau_gate():
    """FB_GATE_TAU_CUM: the updated tokens summed since each head's last recompute,
    on the 8B-dLLM layer (full size): decisions bit-exact, outputs within tolerance,
    and the device count equals the oracle's after the run."""
    w = W.dllm_layer(steps=10)
    gpu, cache = run_policy_gpu(w, flags=W.GATE_TAU_CUM)
    ocache = policy.OracleCache.empty(w.problem)
    ref = policy.run_policy(w, flags=W.GATE_TAU_CUM, cache=ocache)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}: decisions differ"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"cumulative step {s}")
    recs = np.array([r.recompute[0, 0] for r in ref])
    assert recs[0] and recs[1:].any() and not recs[1:].all()
    assert np.array_equal(cache.m_acc.cpu().numpy()[:w.problem.num_seqs], ocache.m_acc)


def test_branch_sync_and_refresh():
    """BlockBatch hooks between steps of the varlen-branch workload: the 64-token
    branch takes the 128-token leader's entries (leader sync), the 4-token branch is
    refreshed.  The copy is bit-exact on the device; later steps match the oracle
    applying the same hooks to its own cache."""
    import dataclasses
    import torch
    from cached_split_attention_b200 import binding as B
    w = W.varlen_branches(steps=4, prefix=512)
    p0 = w.problem
    first = dataclasses.replace(w, steps=w.steps[:2])
    rest = dataclasses.replace(w, steps=w.steps[2:])
    gpu, cache = run_policy_gpu(first)
    ocache = policy.OracleCache.empty(p0)
    policy.run_policy(first, cache=ocache)
    dp = B.DeviceProblem(p0)
    cu = p0.cu_seqlens_kv_in
    src_rows = cache.a_out[cu[5]:cu[5] + (cu[5] - cu[4])].clone()
    src_valid = cache.valid[5].clone()
    mask = torch.zeros(p0.num_seqs, dtype=torch.uint8, device="cuda")
    mask[0] = 1
    B.cache_copy_seq(dp, cache, 5, 4)
    B.cache_invalidate_seqs(dp, cache, mask)
    torch.cuda.synchronize()
    assert torch.equal(cache.a_out[cu[4]:cu[5]], src_rows)
    assert torch.equal(cache.valid[4], src_valid) and not cache.valid[0].any()
    policy.cache_copy_seq(ocache, p0, 5, 4)
    policy.cache_invalidate_seqs(ocache, [b == 0 for b in range(p0.num_seqs)])
    assert np.array_equal(cache.valid.cpu().numpy()[:p0.num_seqs].astype(bool), ocache.valid)
    gpu2, _ = run_policy_gpu(rest, cache=cache)
    ref2 = policy.run_policy(rest, cache=ocache)
    for s, (g, r) in enumerate(zip(gpu2, ref2)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s + 2}: decisions differ"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"after hooks, step {s + 2}")
    assert ref2[0].recompute[0].all()  # the refreshed branch recomputes
