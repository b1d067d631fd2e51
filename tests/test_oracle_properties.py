"""Property tests of the oracle (CPU): facts of softmax attention and of the gates
that hold for any input, drawn by hypothesis.  Each one fails under a plausible
mistake that the fixed pins might let through: a key/value misalignment (key
permutation), a normaliser off by a constant (duplicated keys), a weight outside
[0, 1] (convex hull), a wrong kv-head mapping (GQA equals MHA with repeated kv
heads), a flipped gate comparison (monotonicity in tau and gamma)."""
import math

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from cached_split_attention_b200.workloads import (FORCE_RECOMPUTE, GATE_HEAD, GATE_TAU, make_problem,
                                                   normal_bf16)
from oracle import attention, policy

SETTINGS = settings(max_examples=40, deadline=None)


def _qkv(seed, n, m, d, dv, sharp):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, d)) * sharp, rng.standard_normal((m, d)) * sharp,
            rng.standard_normal((m, dv)))


dims = dict(seed=st.integers(0, 2 ** 31), n=st.integers(1, 6), m=st.integers(1, 12), d=st.integers(1, 9),
            dv=st.integers(1, 5), sharp=st.sampled_from([0.1, 1.0, 4.0]))


@SETTINGS
@given(**dims)
def test_attend_is_invariant_under_key_permutation(seed, n, m, d, dv, sharp):
    q, k, v = _qkv(seed, n, m, d, dv, sharp)
    perm = np.random.default_rng(seed + 1).permutation(m)
    a0, l0 = attention.attend(q, k, v, 1 / math.sqrt(d))
    a1, l1 = attention.attend(q, k[perm], v[perm], 1 / math.sqrt(d))
    assert np.abs(a0 - a1).max() < 1e-12 and np.abs(l0 - l1).max() < 1e-12


@SETTINGS
@given(**dims)
def test_duplicated_keys_keep_a_and_add_ln2_to_l(seed, n, m, d, dv, sharp):
    q, k, v = _qkv(seed, n, m, d, dv, sharp)
    a0, l0 = attention.attend(q, k, v, 0.5)
    a1, l1 = attention.attend(q, np.concatenate([k, k]), np.concatenate([v, v]), 0.5)
    assert np.abs(a0 - a1).max() < 1e-12
    assert np.abs(l1 - (l0 + math.log(2.0))).max() < 1e-12


@SETTINGS
@given(**dims)
def test_output_lies_in_the_convex_hull_of_the_values(seed, n, m, d, dv, sharp):
    q, k, v = _qkv(seed, n, m, d, dv, sharp)
    a, l = attention.attend(q, k, v, 1.0)
    assert np.all(a >= v.min(axis=0) - 1e-12) and np.all(a <= v.max(axis=0) + 1e-12)
    # L is at least the largest score and at most that plus ln m
    s = q @ k.T
    assert np.all(l >= s.max(axis=1) - 1e-12) and np.all(l <= s.max(axis=1) + math.log(m) + 1e-12)


@settings(max_examples=15, deadline=None)
@given(seed=st.integers(0, 2 ** 31), g=st.sampled_from([2, 4]), hkv=st.integers(1, 2),
       which=st.sampled_from(["out", "in"]))
def test_gqa_equals_mha_with_repeated_kv_heads(seed, g, hkv, which):
    rng = np.random.default_rng(seed)
    d = 8
    rows = [np.sort(rng.permutation(6)[:4]), np.arange(3)]
    p = make_problem(rows, [7, 5], [6, 3], g * hkv, hkv, d)
    p_mha = make_problem(rows, [7, 5], [6, 3], g * hkv, g * hkv, d)
    q = normal_bf16(rng, (p.total_q, g * hkv, d))
    tot = p.total_kv_out if which == "out" else p.total_kv_in
    k = normal_bf16(rng, (tot, hkv, d))
    v = normal_bf16(rng, (tot, hkv, d))
    a0, l0 = attention.attend_problem(p, q, k, v, which)
    a1, l1 = attention.attend_problem(p_mha, q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), which)
    assert np.array_equal(a0, a1) and np.array_equal(l0, l1)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), tau=st.integers(0, 8))
def test_tau_gate_is_monotone(seed, tau):
    """A larger tau never turns a reuse into a recompute; tau = 0 reuses nothing."""
    rng = np.random.default_rng(seed)
    valid = rng.random((5, 3)) < 0.8
    n = rng.integers(0, 10, 5)
    r0 = policy.decide(GATE_TAU, tau, 0.0, valid, n)
    r1 = policy.decide(GATE_TAU, tau + 1, 0.0, valid, n)
    assert np.all(r1 <= r0)
    assert policy.decide(GATE_TAU, 0, 0.0, valid, n).all()
    assert np.all(policy.decide(GATE_TAU, 11, 0.0, valid, n) == ~valid)


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), gamma=st.floats(-1.0, 0.99))
def test_gamma_gate_is_monotone(seed, gamma):
    """A larger gamma never turns a recompute into a reuse; gamma >= 1 reuses nothing."""
    rng = np.random.default_rng(seed)
    valid = np.ones((4, 6), dtype=bool)
    cos = rng.uniform(-1, 1, (4, 6))
    r0 = policy.decide(GATE_HEAD, 0, gamma, valid, np.zeros(4), cos=cos)
    r1 = policy.decide(GATE_HEAD, 0, min(gamma + 0.01, 1.0), valid, np.zeros(4), cos=cos)
    assert np.all(r1 >= r0)
    assert policy.decide(GATE_HEAD, 0, 1.0, valid, np.zeros(4), cos=cos).all()
    assert policy.decide(FORCE_RECOMPUTE | GATE_HEAD, 0, -2.0, valid, np.zeros(4), cos=cos).all()
