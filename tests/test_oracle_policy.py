"""The oracle's step policy on the seeded workloads (CPU only)."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from oracle import attention, policy


def test_tiny_policy_decisions_and_fresh_step():
    w = W.tiny()
    res = policy.run_policy(w, with_exact=True)
    assert res[0].recompute.all()                  # no cache yet
    for r in res[1:]:
        assert not r.recompute.any()               # M = 4 < tau = 8
    assert res[0].reuse_error < 1e-12              # fresh cache == full attention
    assert all(r.reuse_error > 0 for r in res[1:])  # reuse is an approximation


def test_dllm_decisions_follow_tau():
    w = W.dllm_layer(steps=12, prefix=256)
    res = policy.run_policy(w)
    for s, r in enumerate(res):
        m = int(w.steps[s].n_updated[0])
        assert 1 <= m <= 4 or s == 0
        expect = True if s == 0 else (m >= 4)
        assert r.recompute.all() == expect and r.recompute.any() == expect


def test_unchanged_queries_make_reuse_exact():
    """Reusing a cache built from the same queries gives bitwise the same result
    as recomputing it (the merge is deterministic in its inputs)."""
    w = W.tiny(steps=3)
    for st in w.steps[1:]:
        st.q = w.steps[0].q.copy()
        st.k_in = w.steps[0].k_in.copy()
        st.v_in = w.steps[0].v_in.copy()
    reuse = policy.run_policy(w, flags=W.FORCE_REUSE)
    recomp = policy.run_policy(w, flags=W.FORCE_RECOMPUTE)
    for a, b in zip(reuse, recomp):
        assert np.array_equal(a.a_full, b.a_full)
        assert np.array_equal(a.l_full, b.l_full)


def test_sampled_rows_match_full_run():
    w = W.varlen_branches(steps=3, prefix=64)
    full = policy.run_policy(w)
    sample = [(b, 0) for b in range(6)] + [(5, 127), (4, 17)]
    samp = policy.run_policy(w, sample=sample)
    for f, s in zip(full, samp):
        assert np.array_equal(f.recompute, s.recompute)
        ok = ~np.isnan(s.l_full)
        assert ok.any()
        # BLAS may block a sub-matrix product differently: equal up to rounding
        assert np.abs(f.a_full[ok] - s.a_full[ok]).max() < 1e-13
        assert np.abs(f.l_full[ok] - s.l_full[ok]).max() < 1e-13


def test_locking_rows_monotone_and_cache_untouched():
    w = W.locking_tiny()
    cache = policy.OracleCache.empty(w.problem)
    res = policy.run_policy(w, cache=cache)
    prev = None
    for r in res:
        p = r.problem
        cur = set((b, int(x)) for b in range(p.num_seqs)
                  for x in p.q_rows[p.cu_seqlens_q[b]:p.cu_seqlens_q[b + 1]])
        if prev is not None:
            assert cur <= prev                     # the active set only shrinks
        prev = cur
        assert r.a_full.shape[0] == p.total_q    # no output for locked rows
    # positions locked at step 1 keep their step-0 cache entries forever
    p0, p1 = w.steps[0].problem, w.steps[1].problem
    c0 = policy.OracleCache.empty(p0)
    w1 = type(w)(w.name, w.problem, w.k_out, w.v_out, w.steps[:1], w.tau, w.gamma, w.flags)
    policy.run_policy(w1, cache=c0)
    locked = sorted(set(policy.cache_rows(p0)) - set(policy.cache_rows(res[-1].problem)))
    assert locked
    assert np.array_equal(cache.a_out[locked], c0.a_out[locked])


def test_video_gamma_margins_are_wide():
    """The seeded noise levels put every cosine far from gamma (decisions are
    insensitive to rounding), and the sigma=0.02 heads reuse while sigma=0.5 heads
    recompute."""
    w = W.video(steps=3, block=96, prefix_blocks=2, heads=8)
    res = policy.run_policy(w)
    assert res[0].recompute.all()
    for r in res[1:]:
        assert np.all(np.abs(r.cos - w.gamma) > 1e-3)
        lo = w.sigma < 0.1
        assert not r.recompute[0, lo].any()
        assert r.recompute[0, ~lo].all()


def test_branch_hooks():
    """Leader sync copies a branch's entries (positions present on both sides, all
    heads) and its validity; a longer destination stays empty; a refresh empties
    only the marked branches; the other rows are untouched."""
    import pins
    pins.check_branch_hooks(policy.cache_copy_seq, policy.cache_invalidate_seqs)


def test_policy_equals_its_cache_free_restatement():
    """run_policy equals the policy restated without a cache (each head's prefix
    partial recomputed from the queries of its last recompute), under the
    cumulative, per-step and similarity gates."""
    import pins
    pins.check_policy_replay(policy.run_policy)
