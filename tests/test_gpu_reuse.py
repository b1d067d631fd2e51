"""The lean reuse pass of fb_step against the oracle (needs a B200).

On a reuse step of a block of at most 128 keys, the work items (sequence,
kv-head, row tile) whose q-heads all reuse the cache take the lean path inside
the streaming kernels: block attention with warp MMA and the merge with the
cached (A_out, L_out) rows (FlashBlock, "Mecanismo Central").  These cases put its
edges under the same tolerances as every other step test: block lengths around
the 32-key slices and 64-key chunks (1 to 128 keys), head dims 64 and 128, grouped
heads up to the largest group the ABI takes (32), a sequence with no active rows,
locked rows, and calls in which some groups reuse while others recompute."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu
from oracle import policy

pytestmark = pytest.mark.gpu


def _workload(blocks, active, prefix, hq, hkv, d, steps=3, seed=5, redraw=2):
    """Sequences with the given block lengths and active block positions; every
    step redraws `redraw` active tokens of each sequence."""
    rng = np.random.default_rng(seed)
    p = W.make_problem(active, [prefix] * len(blocks), blocks, hq, hkv, d)
    k_out = W.normal_bf16(rng, (p.total_kv_out, hkv, d))
    v_out = W.normal_bf16(rng, (p.total_kv_out, hkv, d))
    q_blk = W.normal_bf16(rng, (p.total_kv_in, hq, d))
    k_blk = W.normal_bf16(rng, (p.total_kv_in, hkv, d))
    v_blk = W.normal_bf16(rng, (p.total_kv_in, hkv, d))

    def snap(n):
        idx = np.concatenate([p.cu_seqlens_kv_in[b] + np.asarray(a, dtype=np.int64) for b, a in enumerate(active)]
                             or [np.zeros(0, np.int64)])
        return W.StepInput(q=np.ascontiguousarray(q_blk[idx]), k_in=k_blk.copy(), v_in=v_blk.copy(),
                           n_updated=np.asarray(n, np.int32), problem=p)

    out = [snap([len(a) for a in active])]
    for _ in range(1, steps):
        ns = []
        for b, a in enumerate(active):
            k = min(redraw, len(a))
            toks = p.cu_seqlens_kv_in[b] + rng.choice(np.asarray(a, dtype=np.int64), size=k, replace=False)
            q_blk[toks] = W.normal_bf16(rng, (k, hq, d))
            k_blk[toks] = W.normal_bf16(rng, (k, hkv, d))
            v_blk[toks] = W.normal_bf16(rng, (k, hkv, d))
            ns.append(k)
        out.append(snap(ns))
    return W.Workload("reuse_case", p, k_out, v_out, out, tau=4, gamma=0.0, flags=W.GATE_TAU)


def _compare(w, flags=None, head_reuse_in=None):
    gpu, _ = run_policy_gpu(w, flags=flags, head_reuse_in=head_reuse_in)
    ref = policy.run_policy(w, flags=flags, head_reuse_in=head_reuse_in)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}: decisions differ"
        if w.problem.total_q:
            assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"step {s}")
    return ref


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [1, 5, 31, 32, 33, 64, 65, 100, 128])
def test_block_lengths(block, d):
    """One MHA sequence (4 heads): step 0 fills the cache, steps 1-2 reuse it."""
    w = _workload([block], [np.arange(block)], 70, 4, 4, d)
    ref = _compare(w, flags=W.FORCE_REUSE)
    assert ref[0].recompute.all() and not ref[1].recompute.any()


@pytest.mark.parametrize("g", [2, 4, 8, 16, 32])
def test_grouped_heads_locked_rows(g):
    """GQA groups of g q-heads over 2 kv-heads (tensor-core kernel, up to ten 128-row
    tiles per group); two sequences with locked rows (active positions not the
    identity), blocks of 64 and 47 keys."""
    rng = np.random.default_rng(g)
    active = [np.sort(rng.permutation(64)[:29]), np.sort(rng.permutation(47)[:40])]
    w = _workload([64, 47], active, 150, 2 * g, 2, 128)
    _compare(w, flags=W.FORCE_REUSE)


@pytest.mark.parametrize("d", [64, 128])
def test_largest_group_warp_mma(d):
    """g = 32 with two active tokens per sequence: 64 rows per group, the warp-MMA
    kernel's largest tile; ragged blocks of 8 and 5 keys, locked rows."""
    w = _workload([8, 5], [np.array([1, 6]), np.array([0, 3])], 150, 64, 2, d)
    ref = _compare(w, flags=W.FORCE_REUSE)
    assert ref[0].recompute.all() and not ref[1].recompute.any()


@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 64), (8, 2, 128)], ids=["warp_mma", "tensor_core"])
def test_no_prefix_at_all(hq, hkv, d):
    """Every sequence has an empty prefix (J_out empty, so the cached partial is
    (0, -inf) and the merge gives the block partial itself): both forced arms and
    the tau gate."""
    w = _workload([40, 29], [np.arange(40), np.arange(3, 29, 2)], 0, hq, hkv, d)
    _compare(w, flags=W.FORCE_RECOMPUTE)
    _compare(w, flags=W.FORCE_REUSE)
    _compare(w)


def test_sequence_without_active_rows():
    """A sequence whose rows are all locked has nothing to write; its neighbours
    reuse normally."""
    w = _workload([32, 16, 40], [np.arange(32), np.zeros(0, np.int64), np.arange(3, 40, 2)], 90, 4, 2, 128)
    _compare(w, flags=W.FORCE_REUSE)


def test_groups_reuse_and_recompute_in_one_call():
    """The tau gate per sequence and a caller mask per head: in the same call some
    groups have every head reusing (served by the lean path) and others have at
    least one head recomputing (streamed, all of their heads)."""
    w = _workload([64, 64, 64], [np.arange(64)] * 3, 200, 8, 2, 128, steps=4, redraw=3)
    for s, st in enumerate(w.steps[1:], start=1):   # sequence 1 passes tau = 4 on every step
        st.n_updated[:] = [3, 5, 2]
    ref = _compare(w)
    assert not ref[1].recompute[0].any() and ref[1].recompute[1].all() and not ref[1].recompute[2].any()
    masks = [None]
    rng = np.random.default_rng(3)
    for _ in w.steps[1:]:
        m = np.ones((3, 8), dtype=bool)     # reuse everywhere ...
        m[0, rng.integers(0, 4)] = False    # ... but one head of sequence 0, kv-head 0 recomputes
        m[2, 4 + rng.integers(0, 4)] = False
        masks.append(m)
    _compare(w, head_reuse_in=masks)


def test_tiny_head_dim_64_reuse_steps():
    """The tiny workload (d = 64) at its literal scale: steps 1-3 reuse through the
    lean pass."""
    ref = _compare(W.tiny())
    assert not any(r.recompute.any() for r in ref[1:])
