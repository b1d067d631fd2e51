"""The FlashBlock reuse policy, step by step, in fp64.

Per denoise step s and per (sequence b, q-head h) the policy decides whether the
cached out-of-block partial (A_out, L_out) is reused or recomputed:

  * threshold gate (FlashBlock, "Estrategias de Reutilizacion Adaptativa", first
    bullet): with M the number of block tokens updated at this step, M < tau reuses,
    otherwise the partial is recomputed (strict comparison: M = tau recomputes);
  * per-head gate (same section, second bullet): only heads whose similarity
    exceeds gamma reuse (strict: cos = gamma recomputes).  Reading: the similarity
    is the cosine between the head's current active-row queries and the queries the
    cache was built with (rows x d flattened), because once the prefix K/V are
    fixed A_out depends on the queries alone;
  * locked rows (SureLock, "Mecanismo de Funcionamiento"): a locked row computes no
    query and gets no output, but its K/V stay in the block and are still attended.
    The active set only shrinks.

Cumulative variant of the threshold gate (a reading of "the number of updated
tokens"; the pages count them per step): with GATE_TAU_CUM, M is the number of
block tokens updated since the head's cache was built, i.e. the per-step counts
summed over the steps since the head's last recompute, this step included; a
recompute starts the count again from zero.

Readings taken where the pages are silent: gates combine with AND on "reuse"; a
cache that was never filled (or was invalidated) always recomputes, overriding a
forced reuse; FORCE_RECOMPUTE overrides everything; a caller-supplied per-head
reuse mask replaces the gates; with no gate enabled a valid cache is reused;
a zero similarity denominator gives cos = 0 (recompute).

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

from .attention import attend, attend_full, bf16_to_f64, merge

GATE_TAU = 1
GATE_HEAD = 2
FORCE_RECOMPUTE = 4
FORCE_REUSE = 8
GATE_TAU_CUM = 16


@dataclasses.dataclass
class OracleCache:
    """(A_out, L_out) per block position and q-head, plus bookkeeping.

    a_out [total_kv_in, H_q, d], l_out [total_kv_in, H_q], valid [num_seqs, H_q],
    q_ref [total_kv_in, H_q, d]: the queries each head's cache was built with,
    m_acc [num_seqs, H_q]: block tokens updated since the head's last recompute
    (GATE_TAU_CUM)."""
    a_out: np.ndarray
    l_out: np.ndarray
    valid: np.ndarray
    q_ref: np.ndarray
    m_acc: np.ndarray = None

    @classmethod
    def empty(cls, problem):
        T, H, d = problem.total_kv_in, problem.num_heads_q, problem.head_dim
        return cls(a_out=np.full((T, H, d), np.nan), l_out=np.full((T, H), np.nan),
                   valid=np.zeros((problem.num_seqs, H), dtype=bool),
                   q_ref=np.zeros((T, H, d)), m_acc=np.zeros((problem.num_seqs, H), dtype=np.int64))


def cache_rows(problem) -> np.ndarray:
    """Block-position (cache) row of every packed active row."""
    out = np.empty(problem.total_q, dtype=np.int64)
    for b in range(problem.num_seqs):
        r0, r1 = int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])
        out[r0:r1] = int(problem.cu_seqlens_kv_in[b]) + problem.q_rows[r0:r1]
    return out


def head_cosine(problem, q: np.ndarray, q_ref: np.ndarray) -> np.ndarray:
    """cos[b, h] between current active queries q [total_q, H, d] (fp64) and the
    cached queries q_ref [total_kv_in, H, d] at the same block positions."""
    H = problem.num_heads_q
    crow = cache_rows(problem)
    cos = np.zeros((problem.num_seqs, H))
    for b in range(problem.num_seqs):
        r0, r1 = int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])
        for h in range(H):
            x = q[r0:r1, h].reshape(-1)
            y = q_ref[crow[r0:r1], h].reshape(-1)
            den = np.sqrt(np.dot(x, x) * np.dot(y, y))
            cos[b, h] = np.dot(x, y) / den if den > 0 else 0.0
    return cos


def decide(flags: int, tau: int, gamma: float, valid: np.ndarray, n_updated: np.ndarray,
           cos: Optional[np.ndarray] = None, head_reuse_in: Optional[np.ndarray] = None,
           m_acc: Optional[np.ndarray] = None) -> np.ndarray:
    """recompute[b, h] (bool) from the gate inputs; see the module docstring.
    ``m_acc`` [num_seqs, H_q] is the cumulative count before this step (GATE_TAU_CUM)."""
    valid = np.asarray(valid, dtype=bool)
    S, H = valid.shape
    if flags & FORCE_RECOMPUTE:
        return np.ones((S, H), dtype=bool)
    if flags & FORCE_REUSE:
        reuse = np.ones((S, H), dtype=bool)
    elif head_reuse_in is not None:
        reuse = np.asarray(head_reuse_in, dtype=bool).copy()
    else:
        reuse = np.ones((S, H), dtype=bool)
        if flags & GATE_TAU:
            m = np.asarray(n_updated, dtype=np.int64)
            reuse &= (m < int(tau))[:, None]
        if flags & GATE_TAU_CUM:
            m = np.asarray(m_acc, dtype=np.int64) + np.asarray(n_updated, dtype=np.int64)[:, None]
            reuse &= m < int(tau)
        if flags & GATE_HEAD:
            reuse &= np.asarray(cos) > np.float64(gamma)
    return ~(reuse & valid)


def next_m_acc(flags: int, m_acc: np.ndarray, n_updated: np.ndarray, recompute: np.ndarray) -> np.ndarray:
    """Cumulative count after a step: 0 where the head recomputed, else the old
    count plus this step's updates (kept whenever GATE_TAU_CUM is set)."""
    if not flags & GATE_TAU_CUM:
        return np.asarray(m_acc)
    grown = np.asarray(m_acc, dtype=np.int64) + np.asarray(n_updated, dtype=np.int64)[:, None]
    return np.where(recompute, 0, grown)


def cache_invalidate_seqs(cache: OracleCache, seq_mask) -> None:
    """Refresh of some branches (BlockBatch, "Methodologie : BlockBatch", item 3:
    periodic full-sequence refreshes recompute the K/V of the branches): the
    FlashBlock entries of the marked sequences become empty and their cumulative
    counts restart."""
    m = np.asarray(seq_mask, dtype=bool)
    cache.valid[m] = False
    if cache.m_acc is not None:
        cache.m_acc[m] = 0


def cache_copy_seq(cache: OracleCache, problem, src: int, dst: int) -> None:
    """Leader-based synchronisation (BlockBatch, "Methodologie : BlockBatch", item 2:
    a lagging branch copies the leader's sequence state and K/V cache): the entries
    of block positions 0..min(B_src, B_dst)-1 of every head are copied from sequence
    src to sequence dst, with the validity and count of each head.  When dst has
    more block positions than src, those it cannot fill leave its heads empty."""
    if src == dst:
        return
    s0, s1 = int(problem.cu_seqlens_kv_in[src]), int(problem.cu_seqlens_kv_in[src + 1])
    d0, d1 = int(problem.cu_seqlens_kv_in[dst]), int(problem.cu_seqlens_kv_in[dst + 1])
    n = min(s1 - s0, d1 - d0)
    cache.a_out[d0:d0 + n] = cache.a_out[s0:s0 + n]
    cache.l_out[d0:d0 + n] = cache.l_out[s0:s0 + n]
    cache.q_ref[d0:d0 + n] = cache.q_ref[s0:s0 + n]
    cache.valid[dst] = cache.valid[src] & (d1 - d0 <= s1 - s0)
    if cache.m_acc is not None:
        cache.m_acc[dst] = cache.m_acc[src]


@dataclasses.dataclass
class StepResult:
    recompute: np.ndarray          # [num_seqs, H_q] bool
    cos: Optional[np.ndarray]      # [num_seqs, H_q] or None (gate off)
    a_full: np.ndarray             # [total_q, H_q, d] fp64 (NaN outside the sample)
    l_full: np.ndarray             # [total_q, H_q]
    reuse_error: Optional[float]   # max |A_full - A_exact| over the sample (information only)
    problem: object


def _sample_rows(problem, sample: Optional[Sequence[Tuple[int, int]]]):
    """Packed rows of this step that are in the sample of (seq, block position)."""
    if sample is None:
        return None
    want = set((int(b), int(p)) for b, p in sample)
    rows = []
    for b in range(problem.num_seqs):
        r0, r1 = int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])
        for r in range(r0, r1):
            if (b, int(problem.q_rows[r])) in want:
                rows.append(r)
    return rows


def run_policy(workload, sample: Optional[Sequence[Tuple[int, int]]] = None,
               flags: Optional[int] = None, head_reuse_in: Optional[List[Optional[np.ndarray]]] = None,
               with_exact: bool = False, cache: Optional[OracleCache] = None) -> List[StepResult]:
    """Replay a workload's steps with the FlashBlock cache.

    For each step: decide per (b, h); recompute (A_out, L_out) of the active rows
    of the heads that recompute and store them with their queries; compute the
    in-block partial; merge.  ``sample`` limits the attention work to some
    (sequence, block position) pairs; the gate decisions always use every row."""
    flags = workload.flags if flags is None else flags
    p0 = workload.problem
    cache = cache or OracleCache.empty(p0)
    Hq, Hk = p0.num_heads_q, p0.num_heads_kv
    g = Hq // Hk
    results = []
    for s, st in enumerate(workload.steps):
        p = st.problem
        q = bf16_to_f64(st.q)
        cos = None
        if flags & GATE_HEAD:
            cos = head_cosine(p, q, cache.q_ref)
        hr = None if head_reuse_in is None else head_reuse_in[s]
        if cache.m_acc is None:
            cache.m_acc = np.zeros(cache.valid.shape, dtype=np.int64)
        rec = decide(flags, workload.tau, workload.gamma, cache.valid, st.n_updated, cos, hr, cache.m_acc)
        cache.m_acc = next_m_acc(flags, cache.m_acc, st.n_updated, rec)
        rows = _sample_rows(p, sample)
        crow = cache_rows(p)
        # recompute the out-of-block partial where the gates say so
        for b in range(p.num_seqs):
            r0, r1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
            heads = [h for h in range(Hq) if rec[b, h]]
            if not heads:
                continue
            rs_all = np.arange(r0, r1)
            rs = rs_all if rows is None else np.asarray([r for r in rows if r0 <= r < r1], dtype=np.int64)
            if len(rs):
                o0, o1 = int(p.cu_seqlens_kv_out[b]), int(p.cu_seqlens_kv_out[b + 1])
                for hk in sorted(set(h // g for h in heads)):
                    kk = bf16_to_f64(workload.k_out[o0:o1, hk])
                    vv = bf16_to_f64(workload.v_out[o0:o1, hk])
                    for h in heads:
                        if h // g != hk:
                            continue
                        a, l = attend(q[rs, h], kk, vv, p.softmax_scale)
                        cache.a_out[crow[rs], h] = a
                        cache.l_out[crow[rs], h] = l
            for h in heads:
                cache.q_ref[crow[rs_all], h] = q[rs_all, h]
                cache.valid[b, h] = True
        # in-block partial and merge
        from .attention import attend_problem
        a_in, l_in = attend_problem(p, st.q, st.k_in, st.v_in, "in", rows=rows, q_f64=q)
        a_full, l_full = merge(cache.a_out[crow], cache.l_out[crow], a_in, l_in)
        if rows is not None:
            mask = np.zeros(p.total_q, dtype=bool)
            mask[rows] = True
            a_full[~mask] = np.nan
            l_full[~mask] = np.nan
        err = None
        if with_exact:
            a_ex, _ = attend_full(p, st.q, workload.k_out, workload.v_out, st.k_in, st.v_in, rows=rows)
            sel = slice(None) if rows is None else rows
            err = float(np.nanmax(np.abs(a_full[sel] - a_ex[sel]))) if p.total_q else 0.0
        results.append(StepResult(recompute=rec, cos=cos, a_full=a_full, l_full=l_full,
                                  reuse_error=err, problem=p))
    return results
