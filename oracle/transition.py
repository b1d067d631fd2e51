"""Block transition, in fp64 terms (test infrastructure only).

FlashBlock ("Mecanismo Central") splits the keys a block's queries see into the
tokens outside the block (J_out, stable) and the block's own tokens (J_in).  When a
block is finished, its tokens are no longer being denoised: they become context
for the next block, i.e. part of the next block's J_out.  Reading (the plainest the
pages support): for every sequence b, J_out'(b) = J_out(b) followed by the finished
block's final K/V (those of its last step), in block order; the next block brings
new queries, so no cached (A_out, L_out) applies to them and the cache starts empty
(every head recomputes at the next block's first step).

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

import dataclasses

import numpy as np


def grow_prefix(problem, k_out, v_out, k_in, v_in):
    """J_out'(b) = J_out(b) then J_in(b), for every sequence b.

    Returns (cu_seqlens_kv_out', k_out', v_out'): the new prefix index array and the
    packed K/V (bf16 bits, THD), sequence after sequence."""
    cu_o, cu_i = problem.cu_seqlens_kv_out, problem.cu_seqlens_kv_in
    ks, vs, lens = [], [], []
    for b in range(problem.num_seqs):
        o0, o1 = int(cu_o[b]), int(cu_o[b + 1])
        i0, i1 = int(cu_i[b]), int(cu_i[b + 1])
        ks.append(np.concatenate([k_out[o0:o1], k_in[i0:i1]]))
        vs.append(np.concatenate([v_out[o0:o1], v_in[i0:i1]]))
        lens.append((o1 - o0) + (i1 - i0))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cat = lambda parts, like: np.concatenate(parts) if parts else like[:0]
    return cu, cat(ks, k_out), cat(vs, v_out)


def finish_block(workload):
    """The grown prefix after ``workload``'s block: its prefix followed by the block's
    K/V at the last step (the tokens as they were finally decoded)."""
    last = workload.steps[-1]
    return grow_prefix(last.problem, workload.k_out, workload.v_out, last.k_in, last.v_in)


def next_block_workload(finished, following):
    """The following block's workload with its prefix set to the grown one (the
    following block's generator gives the shapes and its own Q/K/V; its prefix
    lengths must be the grown ones)."""
    cu, k, v = finish_block(finished)
    assert np.array_equal(cu, following.problem.cu_seqlens_kv_out), "prefix lengths of the next block"
    return dataclasses.replace(following, k_out=k, v_out=v)
