"""The two large workloads at their full sizes, in the launch configuration the
library picks for them, against the oracle on sampled rows (needs a B200).

Every row is computed on the GPU; the oracle computes the sampled (sequence,
block position) rows one by one, and the gate decisions for every head."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu
from oracle import policy

pytestmark = pytest.mark.gpu


def _sample_rows(w, per_seq, seed):
    rng = np.random.default_rng(seed)
    p = w.problem
    out = []
    for b in range(p.num_seqs):
        rows = p.q_rows[p.cu_seqlens_q[b]:p.cu_seqlens_q[b + 1]]
        for pos in rng.choice(rows, size=min(per_seq, len(rows)), replace=False):
            out.append((b, int(pos)))
    return out


@pytest.fixture(scope="module")
def gqa_workload():
    return W.long_context_gqa(steps=4)


@pytest.mark.parametrize("arm", [W.FORCE_RECOMPUTE, W.FORCE_REUSE], ids=["recompute", "reuse"])
def test_long_context_gqa_full_size(gqa_workload, arm):
    """batch 8, H_q 32 / H_kv 8, d 128, prefix 32768 (1 GiB of K/V), block 64 with
    32 active rows per sequence; 4 of the 16 steps, both comparison arms."""
    w = gqa_workload
    w.flags = arm
    sample = _sample_rows(w, 2, 7)
    gpu, _ = run_policy_gpu(w)
    ref = policy.run_policy(w, sample=sample)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"gqa {arm} step {s}")


def test_video_full_size():
    """H 40, d 128, block 1560, prefix 9360, 10 steps, cosine gate gamma = 0.95."""
    w = W.video()
    sample = _sample_rows(w, 24, 8)
    gpu, _ = run_policy_gpu(w)
    ref = policy.run_policy(w, sample=sample)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}"
        if r.cos is not None:
            assert np.all(np.abs(r.cos - w.gamma) > 1e-5)
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"video step {s}")
    mixed = [r.recompute.any() and not r.recompute.all() for r in ref[1:]]
    assert any(mixed)
