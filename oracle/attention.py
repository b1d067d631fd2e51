"""Definition of the two attention partials and their log-space merge (fp64).

FlashBlock ("Mecanismo Central") splits the keys seen by the active block's
queries into J_out (tokens outside the block, stable across steps) and J_in (the
block's own tokens, changing).  Each partial is ordinary softmax attention over
its key set plus its log-normaliser L = log Z; the full output is rebuilt by the
log-space composition printed there:

    A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}),
    m = max(L_out, L_in).

Readings taken where the pages are silent:
  * scores are s_j = scale * q.k_j with scale = 1/sqrt(d) unless given;
  * L is the natural log of Z = sum_j e^{s_j}, scale included;
  * the merged normaliser is L_full = m + ln(e^{L_out-m} + e^{L_in-m});
  * an empty key set gives A = 0, L = -inf; merging with a -inf side returns the
    other side; two -inf sides give A = 0, L = -inf;
  * with grouped heads (H_q = g * H_kv), q-head h reads kv-head floor(h / g).

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Softmax attention of rows q [n, d] over keys k [m, d] with values v [m, dv].

    Returns (A [n, dv], L [n]) with A = sum_j softmax_j(s) v_j and L = ln sum_j e^{s_j},
    s_j = scale * q.k_j.  The max is subtracted before exponentiating (this changes
    nothing mathematically, it only keeps e^{.} finite)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, m = q.shape[0], k.shape[0]
    if m == 0:
        return np.zeros((n, v.shape[1])), np.full(n, -np.inf)
    s = scale * (q @ k.T)                      # [n, m]
    mx = s.max(axis=1, keepdims=True)          # [n, 1]
    e = np.exp(s - mx)
    z = e.sum(axis=1)                          # [n]
    a = (e @ v) / z[:, None]
    l = mx[:, 0] + np.log(z)
    return a, l


def merge(a_out: np.ndarray, l_out: np.ndarray, a_in: np.ndarray, l_in: np.ndarray):
    """Log-space composition of two partials (FlashBlock, A_full equation).

    a_*: [..., dv]; l_*: [...].  Returns (A_full, L_full)."""
    a_out = np.asarray(a_out, dtype=np.float64)
    a_in = np.asarray(a_in, dtype=np.float64)
    l_out = np.asarray(l_out, dtype=np.float64)
    l_in = np.asarray(l_in, dtype=np.float64)
    m = np.maximum(l_out, l_in)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w_out = np.where(np.isneginf(l_out), 0.0, np.exp(l_out - m_safe))
    w_in = np.where(np.isneginf(l_in), 0.0, np.exp(l_in - m_safe))
    den = w_out + w_in
    den_safe = np.where(empty, 1.0, den)
    a = (w_out[..., None] * a_out + w_in[..., None] * a_in) / den_safe[..., None]
    a = np.where(empty[..., None], 0.0, a)
    l = np.where(empty, -np.inf, m_safe + np.log(den_safe))
    return a, l


def _key_range(problem, which: str, b: int):
    if which == "out":
        cu = problem.cu_seqlens_kv_out
    elif which == "in":
        cu = problem.cu_seqlens_kv_in
    else:
        raise ValueError(which)
    return int(cu[b]), int(cu[b + 1])


def attend_problem(problem, q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                   which: str, rows: Optional[Sequence[int]] = None, heads: Optional[Sequence[int]] = None,
                   q_f64: Optional[np.ndarray] = None):
    """One partial for every packed active row of a varlen problem.

    q_bits [total_q, H_q, d]; k_bits/v_bits [total_kv_which, H_kv, d] (bf16 bits).
    ``which`` is "out" (J_out, the prefix) or "in" (J_in, the block).  Queries of
    sequence b see exactly the keys of sequence b in that set, with no mask inside
    it (the block is bidirectional).  ``rows`` restricts the computation to some
    packed rows (others are left NaN); ``heads`` to some q-heads.

    Returns (A [total_q, H_q, d], L [total_q, H_q]) in float64."""
    Hq, Hk, d = problem.num_heads_q, problem.num_heads_kv, problem.head_dim
    g = Hq // Hk
    T = problem.total_q
    A = np.full((T, Hq, d), np.nan)
    L = np.full((T, Hq), np.nan)
    q = bf16_to_f64(q_bits) if q_f64 is None else q_f64
    row_set = None if rows is None else np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    head_list = list(range(Hq)) if heads is None else list(heads)
    for b in range(problem.num_seqs):
        r0, r1 = int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])
        if row_set is None:
            rs = np.arange(r0, r1)
        else:
            rs = row_set[(row_set >= r0) & (row_set < r1)]
        if len(rs) == 0:
            continue
        k0, k1 = _key_range(problem, which, b)
        for hk in range(Hk):
            hs = [h for h in head_list if h // g == hk]
            if not hs:
                continue
            kk = bf16_to_f64(k_bits[k0:k1, hk])
            vv = bf16_to_f64(v_bits[k0:k1, hk])
            for h in hs:
                a, l = attend(q[rs, h], kk, vv, problem.softmax_scale)
                A[rs, h] = a
                L[rs, h] = l
    return A, L


def attend_full(problem, q_bits, k_out, v_out, k_in, v_in, rows=None, heads=None):
    """Full attention of each active row over J_out(b) U J_in(b) in one softmax.

    This is the plain definition FlashBlock's split must reproduce when the cache
    is fresh (same Q): the keys of both sets are concatenated and attended once."""
    Hq, Hk, d = problem.num_heads_q, problem.num_heads_kv, problem.head_dim
    g = Hq // Hk
    T = problem.total_q
    A = np.full((T, Hq, d), np.nan)
    L = np.full((T, Hq), np.nan)
    q = bf16_to_f64(q_bits)
    row_set = None if rows is None else np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    head_list = list(range(Hq)) if heads is None else list(heads)
    for b in range(problem.num_seqs):
        r0, r1 = int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])
        rs = np.arange(r0, r1) if row_set is None else row_set[(row_set >= r0) & (row_set < r1)]
        if len(rs) == 0:
            continue
        o0, o1 = _key_range(problem, "out", b)
        i0, i1 = _key_range(problem, "in", b)
        for h in head_list:
            hk = h // g
            kk = np.concatenate([bf16_to_f64(k_out[o0:o1, hk]), bf16_to_f64(k_in[i0:i1, hk])])
            vv = np.concatenate([bf16_to_f64(v_out[o0:o1, hk]), bf16_to_f64(v_in[i0:i1, hk])])
            a, l = attend(q[rs, h], kk, vv, problem.softmax_scale)
            A[rs, h] = a
            L[rs, h] = l
    return A, L
