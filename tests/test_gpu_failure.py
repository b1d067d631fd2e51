"""Failure detection on the device: a bounded wait that runs out (needs a B200).

The attention kernels give every mbarrier wait a limit (about two seconds).  This
test makes one run out -- a self-test kernel waits on a barrier nothing completes
-- and checks that the kernel returned with FB_ERR_TIMEOUT in the status word and
that the context is still usable: the next fb_step call runs and matches the
oracle.  No GPU fault, trap or hang is involved."""
import time

import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu, torch_and_binding
from oracle import policy

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    torch, B = torch_and_binding()
    assert B.device_status() == 0
    t0 = time.time()
    B.selftest_wait_timeout()
    status = B.device_status()  # synchronises
    elapsed = time.time() - t0
    assert status == B.ERR_TIMEOUT, status
    assert 1.0 < elapsed < 30.0, elapsed
    assert B.device_status() == 0  # read and cleared
    w = W.tiny(steps=2)
    gpu, _ = run_policy_gpu(w)
    ref = policy.run_policy(w)
    for g, r in zip(gpu, ref):
        assert np.array_equal(g["decision"], r.recompute)
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, "after the timeout")
