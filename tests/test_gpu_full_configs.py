"""The two large workloads at their full sizes, in the launch configuration the
library picks for them, against the oracle on every row of every step (needs a
B200).

The oracle computes every (row, head) of every step in fp64 (about a minute of
host time per workload); the gate decisions are compared for every head."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu
from oracle import policy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa_workload():
    return W.long_context_gqa()


@pytest.mark.parametrize("arm", [W.FORCE_RECOMPUTE, W.FORCE_REUSE], ids=["recompute", "reuse"])
def test_long_context_gqa_full_size(gqa_workload, arm):
    """batch 8, H_q 32 / H_kv 8, d 128, prefix 32768 (1 GiB of K/V), block 64 with
    32 active rows per sequence; all 16 steps, both comparison arms, every row."""
    w = gqa_workload
    assert len(w.steps) == 16
    gpu, _ = run_policy_gpu(w, flags=arm)
    ref = policy.run_policy(w, flags=arm)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}"
        assert not np.isnan(r.a_full).any()
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"gqa {arm} step {s}")
    if arm == W.FORCE_REUSE:
        assert ref[0].recompute.all() and not any(r.recompute.any() for r in ref[1:])


def test_video_full_size():
    """H 40, d 128, block 1560, prefix 9360, all 10 steps, cosine gate gamma = 0.95,
    every row."""
    w = W.video()
    assert len(w.steps) == 10
    gpu, _ = run_policy_gpu(w)
    ref = policy.run_policy(w)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}"
        if r.cos is not None:
            assert np.all(np.abs(r.cos - w.gamma) > 1e-5)
        assert not np.isnan(r.a_full).any()
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"video step {s}")
    mixed = [r.recompute.any() and not r.recompute.all() for r in ref[1:]]
    assert any(mixed)
