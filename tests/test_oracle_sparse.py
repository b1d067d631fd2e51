"""The sparse-residual partition and policy of the oracle (CPU)."""
import numpy as np

import pins
from cached_split_attention_b200 import workloads as W
from oracle import attention, policy, sparse


def test_partition_pins():
    pins.check_sparse_partition(sparse.rearrange, attention.attend_problem, attention.attend_full, attention.merge)


def test_sparse_workload_every_step_is_full_attention_when_recomputed():
    pins.check_sparse_workload(sparse.sparse_workload, policy.run_policy, attention.attend_full)


def test_sparse_policy_fresh_step_is_dense_and_reuse_is_closer():
    """Step 0 (empty cache) of the sparse-residual policy is full attention; on the
    reuse steps the selected keys are always fresh, so the reuse error stays below
    that of plain FlashBlock on the same workload (information: the pages print no
    figure; here checked on one seeded tiny workload with sharp scores)."""
    w = W.tiny(sharp=6.0, steps=4)
    sel = [list(range(0, 16)) + list(range(192, 256))]  # attention sink + local window
    plain = [r.reuse_error for r in sparse.run_policy(w, with_exact=True)]
    res = [r.reuse_error for r in sparse.run_sparse_residual(w, sel, with_exact=True)]
    assert res[0] < 1e-12 and plain[0] < 1e-12
    assert sum(res[1:]) < sum(plain[1:])
