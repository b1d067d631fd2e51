"""The oracle against what the pages and the mathematics fix (CPU only)."""
import numpy as np
import pytest

import pins
from oracle import attention, policy


def test_bf16_widening():
    pins.check_bf16_widening(attention.bf16_to_f64)


def test_golden_attend():
    pins.check_golden_attend(attention.attend)


def test_brute_force_attend():
    pins.check_brute_force(attention.attend)


def test_closed_forms():
    pins.check_closed_forms(attention.attend)


def test_golden_merge():
    pins.check_golden_merge(attention.merge)


def test_fresh_cache_identity():
    pins.check_fresh_cache_identity(attention.attend, attention.merge)


def test_merge_associative_and_order_independent():
    pins.check_merge_order_independent(attention.attend, attention.merge)


def test_golden_gates():
    pins.check_golden_gates(policy.decide)


def test_cosine():
    pins.check_cosine(policy.head_cosine)


def test_problem_level_vs_brute_force():
    pins.check_problem_vs_brute(attention.attend_problem, attention.merge, attention.attend_full)


def test_cumulative_gate():
    pins.check_cumulative_gate(policy.decide, policy.next_m_acc)
