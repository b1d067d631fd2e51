"""Pure-Python restatement of softmax attention, for pinning the oracle.

Written independently of attention.py: plain loops, math.exp and math.fsum
(exactly rounded sums), no numpy arithmetic.  Only for tiny inputs.

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple


def attend_one(q: Sequence[float], keys: Sequence[Sequence[float]], vals: Sequence[Sequence[float]],
               scale: float) -> Tuple[List[float], float]:
    """(A, L) for one query row; L = log of the sum of exp(scores)."""
    if len(keys) == 0:
        return [0.0] * (len(vals[0]) if vals else 0), -math.inf
    scores = [scale * math.fsum(qi * ki for qi, ki in zip(q, key)) for key in keys]
    top = max(scores)
    w = [math.exp(sc - top) for sc in scores]
    z = math.fsum(w)
    dv = len(vals[0])
    a = [math.fsum(w[j] * vals[j][c] for j in range(len(keys))) / z for c in range(dv)]
    return a, top + math.log(z)


def attend_full_problem(problem, q, k_out, v_out, k_in, v_in):
    """Full attention of every active row over prefix U block of its own sequence.

    q: nested lists [total_q][H_q][d]; k_*/v_*: [tokens][H_kv][d] (floats).
    Returns (A [total_q][H_q][d], L [total_q][H_q])."""
    Hq, Hk = problem.num_heads_q, problem.num_heads_kv
    group = Hq // Hk
    A, L = [], []
    for b in range(problem.num_seqs):
        for r in range(int(problem.cu_seqlens_q[b]), int(problem.cu_seqlens_q[b + 1])):
            arow, lrow = [], []
            for h in range(Hq):
                kv = h // group
                keys, vals = [], []
                for t in range(int(problem.cu_seqlens_kv_out[b]), int(problem.cu_seqlens_kv_out[b + 1])):
                    keys.append(k_out[t][kv])
                    vals.append(v_out[t][kv])
                for t in range(int(problem.cu_seqlens_kv_in[b]), int(problem.cu_seqlens_kv_in[b + 1])):
                    keys.append(k_in[t][kv])
                    vals.append(v_in[t][kv])
                a, l = attend_one(q[r][h], keys, vals, problem.softmax_scale)
                arow.append(a)
                lrow.append(l)
            A.append(arow)
            L.append(lrow)
    return A, L
