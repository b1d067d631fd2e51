"""Sparse-residual FlashBlock, in fp64 (test infrastructure only).

FlashBlock, "Estrategias de Reutilizacion Adaptativa", third bullet: FlashBlock is
orthogonal to sparse attention; the keys a sparse pattern does NOT select are
treated as the out-of-block set and their contribution is cached as a residual,
which makes up for what aggressive sparsification drops.

Reading (the plainest the page supports): per sequence, the sparse pattern selects
some prefix keys; every step attends to the block keys and the selected prefix
keys (the in-block set grows by the selection), and the out-of-block partial
cached by FlashBlock covers the prefix keys left out.  The keys are a partition of
prefix + block, so with a fresh cache the merge is exactly full attention.

This module states the partition (``rearrange``) and runs the ordinary policy on
the rearranged problem; the selection is constant over a block (a new selection
changes the residual set, so the cache must be refilled).
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence

import numpy as np

from .policy import run_policy


def rearrange(problem, k_out, v_out, k_in, v_in, selected: Sequence[Sequence[int]]):
    """Partition the keys of every sequence b: J_in' = block keys of b followed by the
    selected prefix keys (in increasing order), J_out' = the other prefix keys (in
    order).  Returns (problem', k_res, v_res, k_ext, v_ext); problem' keeps the
    query rows and their block positions, which stay positions 0..B_b-1 of J_in'."""
    n_seq = problem.num_seqs
    cu_o, cu_i = problem.cu_seqlens_kv_out, problem.cu_seqlens_kv_in
    res_k, res_v, ext_k, ext_v = [], [], [], []
    out_lens, in_lens = [], []
    for b in range(n_seq):
        o0, o1 = int(cu_o[b]), int(cu_o[b + 1])
        i0, i1 = int(cu_i[b]), int(cu_i[b + 1])
        sel = np.asarray(selected[b], dtype=np.int64)
        if len(sel):
            if np.any(np.diff(sel) <= 0) or sel[0] < 0 or sel[-1] >= o1 - o0:
                raise ValueError(f"sequence {b}: selection must be increasing prefix positions")
        keep = np.ones(o1 - o0, dtype=bool)
        keep[sel] = False
        res_k.append(k_out[o0:o1][keep])
        res_v.append(v_out[o0:o1][keep])
        ext_k.append(np.concatenate([k_in[i0:i1], k_out[o0:o1][sel]]))
        ext_v.append(np.concatenate([v_in[i0:i1], v_out[o0:o1][sel]]))
        out_lens.append(int(keep.sum()))
        in_lens.append((i1 - i0) + len(sel))
    cu = lambda lens: np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    p2 = dataclasses.replace(problem, cu_seqlens_kv_out=cu(out_lens), cu_seqlens_kv_in=cu(in_lens))
    cat = lambda parts, like: (np.concatenate(parts) if parts else like[:0])
    return p2, cat(res_k, k_out), cat(res_v, v_out), cat(ext_k, k_in), cat(ext_v, v_in)


def sparse_workload(workload, selected: Sequence[Sequence[int]]):
    """The workload with every step's keys partitioned by ``rearrange`` (the prefix
    is constant, the block K/V change per step)."""
    steps = []
    p2 = k_res = v_res = None
    for st in workload.steps:
        p2s, k_res, v_res, k_ext, v_ext = rearrange(st.problem, workload.k_out, workload.v_out, st.k_in, st.v_in,
                                                    selected)
        steps.append(dataclasses.replace(st, k_in=k_ext, v_in=v_ext, problem=p2s))
        if p2 is None:
            p2 = p2s
    p0, _, _, _, _ = rearrange(workload.problem, workload.k_out, workload.v_out, workload.steps[0].k_in,
                               workload.steps[0].v_in, selected)
    return dataclasses.replace(workload, name=workload.name + "_sparse", problem=p0, k_out=k_res, v_out=v_res,
                               steps=steps)


def run_sparse_residual(workload, selected: Sequence[Sequence[int]], **kw) -> List:
    """The FlashBlock policy on the sparse-residual partition of the keys."""
    return run_policy(sparse_workload(workload, selected), **kw)
