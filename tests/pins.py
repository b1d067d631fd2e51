"""Pins for the oracle: checks against what the pages and the mathematics fix.

Every check takes the implementation under test as arguments, so that
test_oracle_mutations.py can run the same checks on deliberately broken copies of
the oracle and show that each planted mistake is caught.  A check returns None
when it passes and raises AssertionError otherwise.
"""
from __future__ import annotations

import math

import numpy as np

from golden_loader import load
from oracle import brute

TOL = 1e-12


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    same_inf = (np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b)))
    diff = np.where(same_inf, 0.0, np.abs(a - b))
    assert np.all(np.isfinite(diff)), (what, a, b)
    m = float(diff.max(initial=0.0))
    scale = max(1.0, float(np.abs(np.where(np.isinf(b), 0, b)).max(initial=0.0)))
    assert m <= tol * scale, f"{what}: max diff {m}"


# ---------------------------------------------------------------- definition

def check_bf16_widening(bf16_to_f64):
    """bf16 bit patterns widened to binary64 give the exact values the format
    defines (tests/golden/bf16_bits.txt, derived by hand from the bit layout):
    normals, the smallest subnormal, the largest finite value, signed zero, both
    infinities and NaN; the shape of the input is kept."""
    g = load("bf16_bits.txt")
    bits = g["bits"].astype(np.uint16)
    got = bf16_to_f64(bits)
    assert got.dtype == np.float64, got.dtype
    want = g["values"]
    assert np.array_equal(got, want), (got, want)   # exact: widening must not round
    two_d = bf16_to_f64(bits[:10].reshape(2, 5))
    assert two_d.shape == (2, 5) and np.array_equal(two_d.reshape(-1), want[:10])
    nz = bf16_to_f64(g["neg_zero_bits"].astype(np.uint16))
    assert nz[0] == 0.0 and math.copysign(1.0, float(nz[0])) == -1.0, nz
    assert np.isnan(bf16_to_f64(g["nan_bits"].astype(np.uint16))[0])


def check_golden_attend(attend):
    for name in ("attend_two_keys.txt", "attend_three_keys_scaled.txt"):
        g = load(name)
        d = len(g["q"])
        dv = len(g["A"])
        q = g["q"].reshape(1, d)
        k = g["k"].reshape(-1, d)
        v = g["v"].reshape(-1, dv)
        a, l = attend(q, k, v, float(g["scale"][0]))
        _close(a[0], g["A"], what=name + " A")
        _close(l[0], g["L"][0], what=name + " L")


def check_brute_force(attend, seed=0):
    """Random tiny inputs with n != m != d != dv, mild and sharp scores."""
    rng = np.random.default_rng(seed)
    for (n, m, d, dv, sharp) in [(3, 5, 4, 6, 1.0), (1, 1, 3, 2, 1.0), (4, 7, 2, 3, 6.0), (2, 9, 5, 5, 0.05)]:
        q = rng.standard_normal((n, d)) * sharp
        k = rng.standard_normal((m, d)) * sharp
        v = rng.standard_normal((m, dv))
        scale = 1.0 / math.sqrt(d)
        a, l = attend(q, k, v, scale)
        for i in range(n):
            ab, lb = brute.attend_one(list(q[i]), [list(x) for x in k], [list(x) for x in v], scale)
            _close(a[i], ab, tol=1e-12, what="brute A")
            _close(l[i], lb, tol=1e-12, what="brute L")


def check_closed_forms(attend, seed=1):
    rng = np.random.default_rng(seed)
    d, dv = 6, 4
    # one key: A = v, L = s
    q = rng.standard_normal((3, d)); k = rng.standard_normal((1, d)); v = rng.standard_normal((1, dv))
    a, l = attend(q, k, v, 0.7)
    _close(a, np.repeat(v, 3, axis=0), what="one key A")
    _close(l, 0.7 * (q @ k[0]), what="one key L")
    # all scores equal (q = 0): A = mean(V), L = ln m
    m = 11
    k = rng.standard_normal((m, d)); v = rng.standard_normal((m, dv))
    a, l = attend(np.zeros((2, d)), k, v, 0.3)
    _close(a, np.repeat(v.mean(axis=0, keepdims=True), 2, axis=0), what="uniform A")
    _close(l, np.full(2, math.log(m)), what="uniform L")
    # constant values: A = c
    q = rng.standard_normal((4, d)) * 3
    vc = np.tile(np.array([[1.5, -2.0, 0.25, 7.0]]), (m, 1))
    a, _ = attend(q, k, vc, 0.5)
    _close(a, np.tile(vc[:1], (4, 1)), what="constant V")
    # adding c to every score: A unchanged, L shifted by c
    c = 2.75
    q1 = np.concatenate([q, np.ones((4, 1))], axis=1)
    k1 = np.concatenate([k, np.full((m, 1), c / 0.5)], axis=1)
    a0, l0 = attend(q, k, v, 0.5)
    a1, l1 = attend(q1, k1, v, 0.5)
    _close(a1, a0, what="shift A")
    _close(l1, l0 + c, what="shift L")
    # empty key set: A = 0, L = -inf
    a, l = attend(q, np.zeros((0, d)), np.zeros((0, dv)), 0.5)
    _close(a, np.zeros((4, dv)), what="empty A")
    assert np.all(np.isneginf(l)), "empty L"


# ---------------------------------------------------------------- merge

def check_golden_merge(merge):
    g = load("merge_two_partials.txt")
    a, l = merge(g["a_out"][None], g["l_out"], g["a_in"][None], g["l_in"])
    _close(a[0], g["A"], what="golden merge A")
    _close(l[0], g["L"][0], what="golden merge L")
    g = load("merge_empty_side.txt")
    a, l = merge(g["a_out"][None], g["l_out"], g["a_in"][None], g["l_in"])
    _close(a[0], g["A"], what="empty side A")
    _close(l[0], g["L"][0], what="empty side L")
    a, l = merge(g["a_out"][None], np.array([-np.inf]), g["a_in"][None], np.array([-np.inf]))
    _close(a[0], g["both_A"], what="both empty A")
    assert np.isneginf(l[0]), "both empty L"
    # and symmetrically with the empty side second
    a, l = merge(g["a_in"][None], g["l_in"], g["a_out"][None], g["l_out"])
    _close(a[0], g["A"], what="empty side (swapped) A")


def check_fresh_cache_identity(attend, merge, seed=2):
    """merge(attend(Q, J_out), attend(Q, J_in)) == attend(Q, J_out U J_in)."""
    rng = np.random.default_rng(seed)
    for (n, m1, m2, d, sharp) in [(5, 13, 4, 8, 1.0), (3, 1, 9, 4, 5.0), (2, 30, 30, 16, 0.2)]:
        q = rng.standard_normal((n, d)) * sharp
        k1 = rng.standard_normal((m1, d)); v1 = rng.standard_normal((m1, 3))
        k2 = rng.standard_normal((m2, d)) * sharp; v2 = rng.standard_normal((m2, 3))
        s = 1 / math.sqrt(d)
        ao, lo = attend(q, k1, v1, s)
        ai, li = attend(q, k2, v2, s)
        a, l = merge(ao, lo, ai, li)
        af, lf = attend(q, np.concatenate([k1, k2]), np.concatenate([v1, v2]), s)
        _close(a, af, what="fresh identity A")
        _close(l, lf, what="fresh identity L")


def check_merge_order_independent(attend, merge, seed=3):
    """Any partition of the keys into 2..16 chunks, merged in any order and tree
    shape, gives the same (A, L) as one attention over all keys."""
    rng = np.random.default_rng(seed)
    n, m, d = 4, 64, 8
    q = rng.standard_normal((n, d)) * 2
    k = rng.standard_normal((m, d)); v = rng.standard_normal((m, 5))
    s = 1 / math.sqrt(d)
    af, lf = attend(q, k, v, s)
    for trial in range(12):
        nchunks = int(rng.integers(2, 17))
        cuts = np.sort(rng.choice(np.arange(1, m), size=nchunks - 1, replace=False))
        bounds = np.concatenate([[0], cuts, [m]])
        parts = [attend(q, k[a:b], v[a:b], s) for a, b in zip(bounds[:-1], bounds[1:])]
        # include an empty chunk now and then
        if trial % 3 == 0:
            parts.append(attend(q, k[:0], v[:0], s))
        order = rng.permutation(len(parts))
        parts = [parts[i] for i in order]
        while len(parts) > 1:                     # random tree shape
            i = int(rng.integers(0, len(parts) - 1))
            (a1, l1), (a2, l2) = parts[i], parts[i + 1]
            parts[i:i + 2] = [merge(a1, l1, a2, l2)]
        a, l = parts[0]
        _close(a, af, tol=1e-11, what="tree merge A")
        _close(l, lf, tol=1e-11, what="tree merge L")
    # commutativity, exactly
    a1, l1 = attend(q, k[:20], v[:20], s)
    a2, l2 = attend(q, k[20:], v[20:], s)
    x = merge(a1, l1, a2, l2)
    y = merge(a2, l2, a1, l1)
    _close(x[0], y[0], tol=1e-15, what="commutative A")
    _close(x[1], y[1], tol=1e-15, what="commutative L")


# ---------------------------------------------------------------- gates

def check_golden_gates(decide):
    g = load("gates.txt")
    tc = g["tau_cases"].reshape(-1, 3)
    for tau, m, exp in tc:
        rec = decide(1, int(tau), 0.0, np.ones((1, 1), bool), np.array([int(m)]), None, None)
        assert bool(rec[0, 0]) == bool(exp), ("tau", tau, m, exp)
    gc = g["gamma_cases"].reshape(-1, 3)
    for gamma, cos, exp in gc:
        rec = decide(2, 0, float(gamma), np.ones((1, 1), bool), np.array([0]), np.array([[cos]]), None)
        assert bool(rec[0, 0]) == bool(exp), ("gamma", gamma, cos, exp)
    # an invalid cache always recomputes, even under forced reuse
    rec = decide(8, 0, 0.0, np.zeros((1, 2), bool), np.array([0]), None, None)
    assert rec.all(), "invalid cache must recompute"
    rec = decide(4, 100, 0.0, np.ones((1, 2), bool), np.array([0]), None, None)
    assert rec.all(), "force recompute"
    rec = decide(8 | 1, 4, 0.0, np.ones((1, 2), bool), np.array([99]), None, None)
    assert not rec.any(), "force reuse overrides a failing tau gate"
    # both gates: AND on reuse
    rec = decide(3, 4, 0.5, np.ones((2, 2), bool), np.array([3, 3]), np.array([[0.9, 0.1], [0.6, 0.7]]), None)
    assert rec.tolist() == [[False, True], [False, False]], rec
    rec = decide(3, 4, 0.5, np.ones((1, 2), bool), np.array([4]), np.array([[0.9, 0.9]]), None)
    assert rec.all(), "tau failure must recompute regardless of cos"


def check_cumulative_gate(decide, next_m_acc):
    """The GATE_TAU_CUM sequence of tests/golden/gates.txt, step by step; plus the
    per-sequence broadcast of n_updated over heads and the reset on any recompute."""
    g = load("gates.txt")
    tau = int(g["cum_tau"][0])
    steps = g["cum_steps"].reshape(-1, 3)
    valid = np.zeros((1, 1), bool)
    m_acc = np.zeros((1, 1), np.int64)
    for s, (n, exp_rec, exp_m) in enumerate(steps):
        rec = decide(16, tau, 0.0, valid, np.array([int(n)]), None, None, m_acc)
        assert bool(rec[0, 0]) == bool(exp_rec), ("cumulative step", s, rec, exp_rec)
        m_acc = next_m_acc(16, m_acc, np.array([int(n)]), rec)
        assert int(m_acc[0, 0]) == int(exp_m), ("cumulative count", s, m_acc, exp_m)
        valid = valid | rec
    # two sequences x two heads: counts differ per head, updates per sequence
    m_acc = np.array([[0, 3], [2, 1]])
    rec = decide(16, 4, 0.0, np.ones((2, 2), bool), np.array([1, 2]), None, None, m_acc)
    assert rec.tolist() == [[False, True], [True, False]], rec
    nxt = next_m_acc(16, m_acc, np.array([1, 2]), rec)
    assert nxt.tolist() == [[1, 0], [0, 3]], nxt
    # a forced recompute resets the count; a caller mask replaces the gate
    rec = decide(16 | 4, 4, 0.0, np.ones((1, 1), bool), np.array([0]), None, None, np.array([[1]]))
    assert rec.all() and next_m_acc(16, np.array([[1]]), np.array([0]), rec).tolist() == [[0]]
    # without the flag the count is not kept
    assert next_m_acc(1, np.array([[5]]), np.array([3]), np.array([[False]])).tolist() == [[5]]


def check_cosine(head_cosine):
    """cos(x, x) = 1, cos(x, -x) = -1, cos(x, 2x) = 1, orthogonal rows = 0, over the
    active rows of each sequence only (cache rows addressed by block position)."""
    from cached_split_attention_b200.workloads import make_problem
    p = make_problem([[0, 2], [1]], [3, 3], [3, 2], 2, 1, 4)
    q = np.zeros((3, 2, 4))
    q_ref = np.zeros((5, 2, 4))
    # seq 0 rows at block positions 0 and 2 -> cache rows 0 and 2
    x = np.array([[1.0, 2.0, 0.0, -1.0], [0.5, 0.0, 3.0, 1.0]])
    q[0:2, 0] = x
    q_ref[[0, 2], 0] = x
    q[0:2, 1] = x
    q_ref[[0, 2], 1] = -2.0 * x
    q_ref[1, 0] = 100.0            # an inactive position: must be ignored
    # seq 1: row at block position 1 -> cache row 3 + 1 = 4
    q[2, 0] = [1, 0, 0, 0]
    q_ref[4, 0] = [0, 1, 0, 0]
    q[2, 1] = [1, 1, 0, 0]
    q_ref[4, 1] = [3, 3, 0, 0]
    cos = head_cosine(p, q, q_ref)
    _close(cos, np.array([[1.0, -1.0], [0.0, 1.0]]), tol=1e-15, what="cosine")


# ---------------------------------------------------------------- problem-level

def check_problem_vs_brute(attend_problem, merge, attend_full_fn=None, seed=4):
    """A GQA varlen problem (3 sequences, ragged, one with an empty prefix): the
    split partials merged must equal brute-force full attention over J_out U J_in."""
    from cached_split_attention_b200.workloads import make_problem, normal_bf16
    from oracle.attention import bf16_to_f64
    rng = np.random.default_rng(seed)
    Hq, Hk, d = 4, 2, 8
    p = make_problem([[0, 1, 2], [1, 3], [0]], [5, 0, 3], [3, 4, 2], Hq, Hk, d)
    q = normal_bf16(rng, (p.total_q, Hq, d), 1.5)
    ko = normal_bf16(rng, (p.total_kv_out, Hk, d)); vo = normal_bf16(rng, (p.total_kv_out, Hk, d))
    ki = normal_bf16(rng, (p.total_kv_in, Hk, d)); vi = normal_bf16(rng, (p.total_kv_in, Hk, d))
    ao, lo = attend_problem(p, q, ko, vo, "out")
    ai, li = attend_problem(p, q, ki, vi, "in")
    a, l = merge(ao, lo, ai, li)
    tolist = lambda x: bf16_to_f64(x).tolist()
    ab, lb = brute.attend_full_problem(p, tolist(q), tolist(ko), tolist(vo), tolist(ki), tolist(vi))
    _close(a, np.array(ab), what="problem A")
    _close(l, np.array(lb), what="problem L")
    if attend_full_fn is not None:
        af, lf = attend_full_fn(p, q, ko, vo, ki, vi)
        _close(af, np.array(ab), what="attend_full A")
        _close(lf, np.array(lb), what="attend_full L")


def _sparse_case(seed=3):
    """Two sequences (GQA 4/2, d = 16), prefixes 40 and 23, blocks 12 and 9 (a few
    rows locked), bf16 inputs with sharp scores."""
    from cached_split_attention_b200.workloads import make_problem, normal_bf16
    rng = np.random.default_rng(seed)
    p = make_problem([[0, 3, 4, 7, 11], [1, 2, 8]], [40, 23], [12, 9], 4, 2, 16)
    q = normal_bf16(rng, (p.total_q, 4, 16), 0.6)
    ko = normal_bf16(rng, (p.total_kv_out, 2, 16), 0.6)
    vo = normal_bf16(rng, (p.total_kv_out, 2, 16))
    ki = normal_bf16(rng, (p.total_kv_in, 2, 16), 0.6)
    vi = normal_bf16(rng, (p.total_kv_in, 2, 16))
    return p, q, ko, vo, ki, vi


def check_sparse_partition(rearrange, attend_problem, attend_full, merge):
    """The sparse-residual partition (FlashBlock, "Estrategias de Reutilizacion
    Adaptativa", third bullet) is a partition of each sequence's keys: the rows of
    J_out' and J_in' are those of prefix + block, once each; the block stays at
    positions 0..B-1 of J_in'; with a fresh cache the merge of the two partials is
    full attention over prefix + block; an empty selection changes nothing."""
    p, q, ko, vo, ki, vi = _sparse_case()
    for sel in ([[0, 5, 6, 39], [22]], [[], list(range(23))], [list(range(40)), []]):
        p2, kr, vr, ke, ve = rearrange(p, ko, vo, ki, vi, sel)
        for b in range(p.num_seqs):
            orig = np.concatenate([ko[p.cu_seqlens_kv_out[b]:p.cu_seqlens_kv_out[b + 1]],
                                   ki[p.cu_seqlens_kv_in[b]:p.cu_seqlens_kv_in[b + 1]]])
            orig_v = np.concatenate([vo[p.cu_seqlens_kv_out[b]:p.cu_seqlens_kv_out[b + 1]],
                                     vi[p.cu_seqlens_kv_in[b]:p.cu_seqlens_kv_in[b + 1]]])
            new = np.concatenate([kr[p2.cu_seqlens_kv_out[b]:p2.cu_seqlens_kv_out[b + 1]],
                                  ke[p2.cu_seqlens_kv_in[b]:p2.cu_seqlens_kv_in[b + 1]]])
            new_v = np.concatenate([vr[p2.cu_seqlens_kv_out[b]:p2.cu_seqlens_kv_out[b + 1]],
                                    ve[p2.cu_seqlens_kv_in[b]:p2.cu_seqlens_kv_in[b + 1]]])
            key = lambda k, v: sorted(map(bytes, np.concatenate([k.reshape(len(k), -1), v.reshape(len(v), -1)], 1)))
            assert key(orig, orig_v) == key(new, new_v), ("keys not a partition", b)
            i0, i0n = int(p.cu_seqlens_kv_in[b]), int(p2.cu_seqlens_kv_in[b])
            nb = int(p.cu_seqlens_kv_in[b + 1]) - i0
            assert np.array_equal(ke[i0n:i0n + nb], ki[i0:i0 + nb]), ("block moved", b)
        assert np.array_equal(p2.q_rows, p.q_rows) and np.array_equal(p2.cu_seqlens_q, p.cu_seqlens_q)
        a_o, l_o = attend_problem(p2, q, kr, vr, "out")
        a_i, l_i = attend_problem(p2, q, ke, ve, "in")
        a, l = merge(a_o, l_o, a_i, l_i)
        a_ex, l_ex = attend_full(p, q, ko, vo, ki, vi)
        assert np.abs(a - a_ex).max() < 1e-12 and np.abs(l - l_ex).max() < 1e-12, "fresh partition is not exact"
    p2, kr, vr, ke, ve = rearrange(p, ko, vo, ki, vi, [[], []])
    assert np.array_equal(kr, ko) and np.array_equal(ve, vi) and np.array_equal(p2.cu_seqlens_kv_in, p.cu_seqlens_kv_in)


def check_sparse_workload(sparse_workload, run_policy, attend_full):
    """The sparse-residual workload, step by step: with FORCE_RECOMPUTE every step
    merges a fresh residual partial (the prefix keys left out) with the partial over
    the block and the selected keys, so at every step the result must be full
    attention over prefix + block of that step's inputs (FlashBlock, "Estrategias de
    Reutilizacion Adaptativa", third bullet, with "Mecanismo Central").  The block
    K/V change at every step, so a rearrangement that kept an old block's keys
    fails from step 1 on.  Run on the tiny workload (one sequence, sharp scores) and
    on the locking workload (two sequences, GQA, shrinking active sets)."""
    from cached_split_attention_b200 import workloads as W
    cases = [(W.tiny(sharp=6.0, steps=4), [list(range(0, 16)) + [77, 130] + list(range(192, 256))]),
             (W.locking_tiny(steps=3), [[0, 5, 6, 40, 95], list(range(20, 60))])]
    for w, sel in cases:
        assert any(not np.array_equal(st.k_in, w.steps[0].k_in) for st in w.steps[1:]), "block must change"
        got = run_policy(sparse_workload(w, sel), flags=W.FORCE_RECOMPUTE)
        for s, (r, st) in enumerate(zip(got, w.steps)):
            a_ex, l_ex = attend_full(st.problem, st.q, w.k_out, w.v_out, st.k_in, st.v_in)
            _close(r.a_full, a_ex, what=f"{w.name} sparse step {s} A")
            _close(r.l_full, l_ex, what=f"{w.name} sparse step {s} L")


# ---------------------------------------------------------------- block transition

def _transition_case():
    """Block 1: two sequences (GQA 4/2, d = 16), prefixes 37 and 0, blocks 20 and 9
    with a few locked rows, 3 steps that redraw tokens; block 2: the block after it."""
    from cached_split_attention_b200 import workloads as W
    rng = np.random.default_rng(11)
    p = W.make_problem([[0, 2, 3, 7, 8, 11, 19], [0, 1, 4, 8]], [37, 0], [20, 9], 4, 2, 16)
    k_out = W.normal_bf16(rng, (p.total_kv_out, 2, 16), 0.7)
    v_out = W.normal_bf16(rng, (p.total_kv_out, 2, 16))
    st = W._BlockState(rng, p, 0.7, 0.7, 1.0)
    steps = [st.step_input([20, 9])]
    for _ in range(2):
        st.redraw(np.array([2, 11, 20 + 4]))
        steps.append(st.step_input([2, 1]))
    w1 = W.Workload("transition_case", p, k_out, v_out, steps, tau=2, gamma=0.0, flags=W.GATE_TAU)
    return w1, W.next_block(w1, seed=12, steps=3, redraws=1)


def check_block_transition(grow_prefix, finish_block, next_block_workload, run_policy, attend):
    """Block transition (FlashBlock, "Mecanismo Central": the finished block's tokens
    leave J_in and become context, i.e. J_out of the next block).
    1. A hand-made case: prefixes of lengths 2 and 0, blocks of 1 and 2 tokens with
       distinct values: J_out' = [p0 p1 b0] and [b1 b2], cu = [0, 3, 5].
    2. The grown prefix is the finished block's *last* step K/V after each prefix.
    3. The next block's first step (empty cache) equals attention of its queries over
       the old prefix, the finished block's final K/V and the new block's K/V,
       concatenated here by hand per sequence and head."""
    from cached_split_attention_b200.workloads import make_problem
    p = make_problem([[0], [0, 1]], [2, 0], [1, 2], 1, 1, 1)
    ko = np.array([[[1]], [[2]]], dtype=np.uint16); vo = ko + 100
    ki = np.array([[[10]], [[11]], [[12]]], dtype=np.uint16); vi = ki + 100
    cu, k2, v2 = grow_prefix(p, ko, vo, ki, vi)
    assert list(cu) == [0, 3, 5], cu
    assert k2.reshape(-1).tolist() == [1, 2, 10, 11, 12], k2.reshape(-1)
    assert v2.reshape(-1).tolist() == [101, 102, 110, 111, 112], v2.reshape(-1)

    from oracle.attention import bf16_to_f64
    w1, nxt = _transition_case()
    cu, k2, v2 = finish_block(w1)
    last = w1.steps[-1]
    assert not np.array_equal(last.k_in, w1.steps[0].k_in), "the case must redraw"
    pl = last.problem
    for b in range(pl.num_seqs):
        o0, o1 = int(pl.cu_seqlens_kv_out[b]), int(pl.cu_seqlens_kv_out[b + 1])
        i0, i1 = int(pl.cu_seqlens_kv_in[b]), int(pl.cu_seqlens_kv_in[b + 1])
        n0 = int(cu[b])
        assert int(cu[b + 1]) - n0 == (o1 - o0) + (i1 - i0)
        assert np.array_equal(k2[n0:n0 + o1 - o0], w1.k_out[o0:o1])
        assert np.array_equal(k2[n0 + o1 - o0:int(cu[b + 1])], last.k_in[i0:i1])
        assert np.array_equal(v2[n0 + o1 - o0:int(cu[b + 1])], last.v_in[i0:i1])
    w2 = next_block_workload(w1, nxt)
    r0 = run_policy(w2)[0]
    st2 = w2.steps[0]
    p2 = st2.problem
    g = p2.num_heads_q // p2.num_heads_kv
    q = bf16_to_f64(st2.q)
    for b in range(p2.num_seqs):
        r_0, r_1 = int(p2.cu_seqlens_q[b]), int(p2.cu_seqlens_q[b + 1])
        o0, o1 = int(pl.cu_seqlens_kv_out[b]), int(pl.cu_seqlens_kv_out[b + 1])
        i0, i1 = int(pl.cu_seqlens_kv_in[b]), int(pl.cu_seqlens_kv_in[b + 1])
        j0, j1 = int(p2.cu_seqlens_kv_in[b]), int(p2.cu_seqlens_kv_in[b + 1])
        for h in range(p2.num_heads_q):
            hk = h // g
            kk = np.concatenate([w1.k_out[o0:o1, hk], last.k_in[i0:i1, hk], st2.k_in[j0:j1, hk]])
            vv = np.concatenate([w1.v_out[o0:o1, hk], last.v_in[i0:i1, hk], st2.v_in[j0:j1, hk]])
            a, l = attend(q[r_0:r_1, h], bf16_to_f64(kk), bf16_to_f64(vv), p2.softmax_scale)
            _close(r0.a_full[r_0:r_1, h], a, what=f"next block step 0 A (seq {b}, head {h})")
            _close(r0.l_full[r_0:r_1, h], l, what=f"next block step 0 L (seq {b}, head {h})")
    assert r0.recompute.all()


# ---------------------------------------------------------------- branch hooks

def check_branch_hooks(cache_copy_seq, cache_invalidate_seqs):
    """BlockBatch, "Methodologie : BlockBatch", items 2 and 3.  Leader sync copies the
    entries of the block positions both branches have, for every head, with the
    leader's validity and count; a destination with more positions than the leader
    stays empty; a refresh empties only the marked branches and restarts their
    counts; nothing else changes."""
    from cached_split_attention_b200.workloads import make_problem
    from oracle import policy
    p = make_problem([[0, 1, 2], [0, 1], [0, 1, 2, 3]], [5, 5, 5], [3, 2, 4], 2, 1, 4)
    c = policy.OracleCache.empty(p)
    rng = np.random.default_rng(0)
    c.a_out[:] = rng.normal(size=c.a_out.shape)
    c.l_out[:] = rng.normal(size=c.l_out.shape)
    c.q_ref[:] = rng.normal(size=c.q_ref.shape)
    c.valid[:] = [[True, False], [True, True], [False, True]]
    c.m_acc[:] = [[1, 2], [3, 4], [5, 6]]
    before = (c.a_out.copy(), c.l_out.copy(), c.q_ref.copy())
    cache_copy_seq(c, p, 0, 1)          # B_src = 3 >= B_dst = 2
    assert np.array_equal(c.a_out[3:5], before[0][0:2]) and np.array_equal(c.l_out[3:5], before[1][0:2])
    assert np.array_equal(c.q_ref[3:5], before[2][0:2])
    assert c.valid[1].tolist() == [True, False] and c.m_acc[1].tolist() == [1, 2]
    assert np.array_equal(c.a_out[0:3], before[0][0:3]) and np.array_equal(c.a_out[5:], before[0][5:])
    assert np.array_equal(c.l_out[0:3], before[1][0:3]) and np.array_equal(c.q_ref[0:3], before[2][0:3])
    cache_copy_seq(c, p, 1, 2)          # B_src = 2 < B_dst = 4: dst cannot be filled
    assert np.array_equal(c.a_out[5:7], before[0][0:2]) and np.array_equal(c.a_out[7:9], before[0][7:9])
    assert not c.valid[2].any()
    cache_invalidate_seqs(c, [True, False, False])
    assert not c.valid[0].any() and c.m_acc[0].tolist() == [0, 0] and c.valid[1].tolist() == [True, False]
    assert c.m_acc[1].tolist() == [1, 2]


# ---------------------------------------------------------------- the step policy

def _replay_expected(w, flags):
    """The FlashBlock policy restated without a cache: a head recomputes at the first
    step and whenever its gate says so; the prefix partial it uses at step s is the
    attention, over the prefix, of the queries it had at its last recompute (same
    block positions); the output merges that with the attention of the current
    queries over the current block (FlashBlock, "Mecanismo Central" and "Estrategias
    de Reutilizacion Adaptativa")."""
    from oracle import attention
    from cached_split_attention_b200.workloads import GATE_HEAD, GATE_TAU, GATE_TAU_CUM
    p0 = w.problem
    S, H, Hk = p0.num_seqs, p0.num_heads_q, p0.num_heads_kv
    g = H // Hk
    last = np.full((S, H), -1)
    count = np.zeros((S, H), dtype=np.int64)
    qs, where = [], []   # per step: queries (fp64) and {(b, block position): packed row}
    decisions, outs = [], []
    for s, st in enumerate(w.steps):
        p = st.problem
        q = attention.bf16_to_f64(st.q)
        qs.append(q)
        where.append({(b, int(p.q_rows[r])): r for b in range(S)
                      for r in range(int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1]))})
        rec = np.zeros((S, H), dtype=bool)
        for b in range(S):
            r0, r1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
            n = int(st.n_updated[b])
            for h in range(H):
                if last[b, h] < 0:
                    rec[b, h] = True
                elif flags & GATE_TAU:
                    rec[b, h] = n >= w.tau
                elif flags & GATE_TAU_CUM:
                    rec[b, h] = count[b, h] + n >= w.tau
                elif flags & GATE_HEAD:
                    then = [where[last[b, h]][(b, int(p.q_rows[r]))] for r in range(r0, r1)]
                    x = q[r0:r1, h].ravel()
                    y = qs[last[b, h]][then, h].ravel()
                    den = math.sqrt(float(x @ x) * float(y @ y))
                    cos = float(x @ y) / den if den > 0 else 0.0
                    rec[b, h] = not (cos > w.gamma)
            if flags & GATE_TAU_CUM:
                count[b] = np.where(rec[b], 0, count[b] + n)
        last[rec] = s
        a_full = np.full((p.total_q, H, p.head_dim), np.nan)
        l_full = np.full((p.total_q, H), np.nan)
        for b in range(S):
            r0, r1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
            if r1 == r0:
                continue
            o0, o1 = int(p.cu_seqlens_kv_out[b]), int(p.cu_seqlens_kv_out[b + 1])
            i0, i1 = int(p.cu_seqlens_kv_in[b]), int(p.cu_seqlens_kv_in[b + 1])
            for h in range(H):
                then = [where[last[b, h]][(b, int(p.q_rows[r]))] for r in range(r0, r1)]
                ko = attention.bf16_to_f64(w.k_out[o0:o1, h // g])
                vo = attention.bf16_to_f64(w.v_out[o0:o1, h // g])
                ki = attention.bf16_to_f64(st.k_in[i0:i1, h // g])
                vi = attention.bf16_to_f64(st.v_in[i0:i1, h // g])
                ao, lo = attention.attend(qs[last[b, h]][then, h], ko, vo, p.softmax_scale)
                ai, li = attention.attend(q[r0:r1, h], ki, vi, p.softmax_scale)
                a, l = attention.merge(ao, lo, ai, li)
                a_full[r0:r1, h] = a
                l_full[r0:r1, h] = l
        decisions.append(rec)
        outs.append((a_full, l_full))
    return decisions, outs


def check_policy_replay(run_policy):
    """run_policy against the cache-free restatement above, on a cumulative-τ problem
    with monotone locking (GQA), a τ-gated problem and a γ-gated problem: decisions
    equal, outputs within 1e-12, and both reuse and recompute taken after step 0."""
    from cached_split_attention_b200 import workloads as W
    locking = W.locking_tiny()
    locking.tau = 7       # 3 redraws per step: the count passes 7 at the third step
    cases = [(locking, W.GATE_TAU_CUM),
             (W.dllm_layer(steps=8, prefix=128), W.GATE_TAU),
             (W.video(steps=4, block=48, prefix_blocks=2, heads=4, head_dim=64, sigma_lo=0.02, sigma_hi=0.6),
              W.GATE_HEAD)]
    for w, flags in cases:
        got = run_policy(w, flags=flags)
        dec, outs = _replay_expected(w, flags)
        for s, (r, d, (a, l)) in enumerate(zip(got, dec, outs)):
            assert np.array_equal(r.recompute, d), (w.name, s, "decisions")
            _close(r.a_full, a, what=f"{w.name} step {s} A")
            _close(r.l_full, l, what=f"{w.name} step {s} L")
        assert any(d.any() for d in dec[1:]) and any((~d).any() for d in dec[1:]), (w.name, "both branches taken")
