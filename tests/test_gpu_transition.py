"""Block transition on the GPU against the oracle (needs a B200).

An episode of two blocks: block 1 runs its steps through fb_step; the block is
finished, so fb_prefix_append builds each sequence's grown prefix (its old prefix,
then the block's final K/V) on the device -- in new buffers, or in place for one
sequence -- and fb_cache_invalidate empties the cache; block 2 (new queries, same
block shapes) then runs on the grown prefix, with new TMA descriptors for the new
buffers.  The grown prefix and its index array must equal the oracle's bit for bit
(FlashBlock, "Mecanismo Central": the finished block's tokens become out-of-block
context), and every step of block 2 must match the oracle's policy on it."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu, torch_and_binding
from oracle import policy, transition

pytestmark = pytest.mark.gpu


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _two_blocks(w1, nxt, in_place=False):
    torch, B = torch_and_binding()
    gpu1, cache = run_policy_gpu(w1)
    ocache = policy.OracleCache.empty(w1.problem)
    ref1 = policy.run_policy(w1, cache=ocache)
    for s, (g, r) in enumerate(zip(gpu1, ref1)):
        assert np.array_equal(g["decision"], r.recompute), f"block 1 step {s}"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"block 1 step {s}")

    last = w1.steps[-1]
    pl = last.problem
    dp = B.DeviceProblem(pl)
    grown = pl.total_kv_out + pl.total_kv_in
    shape = (grown,) + w1.k_out.shape[1:]
    k_in, v_in = B.bf16_tensor(last.k_in), B.bf16_tensor(last.v_in)
    if in_place:   # one buffer with room for the block after the prefix
        k_dst = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        v_dst = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        k_dst[:pl.total_kv_out] = B.bf16_tensor(w1.k_out)
        v_dst[:pl.total_kv_out] = B.bf16_tensor(w1.v_out)
        k_src, v_src = k_dst, v_dst
    else:
        k_src, v_src = B.bf16_tensor(w1.k_out), B.bf16_tensor(w1.v_out)
        k_dst = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        v_dst = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    cu_dst = torch.full((pl.num_seqs + 1,), -7, dtype=torch.int32, device="cuda")
    B.prefix_append(dp, k_src, v_src, k_in, v_in, k_dst, v_dst, cu_dst)
    B.cache_invalidate(dp, cache)
    policy.cache_invalidate_seqs(ocache, np.ones(pl.num_seqs, dtype=bool))
    torch.cuda.synchronize()

    cu_o, k_o, v_o = transition.finish_block(w1)
    assert np.array_equal(cu_dst.cpu().numpy(), cu_o), "grown prefix offsets"
    assert np.array_equal(_bits(k_dst), k_o) and np.array_equal(_bits(v_dst), v_o), "grown prefix K/V"

    w2 = transition.next_block_workload(w1, nxt)
    gpu2, _ = run_policy_gpu(w2, cache=cache, k_out=k_dst, v_out=v_dst)
    ref2 = policy.run_policy(w2, cache=ocache)
    for s, (g, r) in enumerate(zip(gpu2, ref2)):
        assert np.array_equal(g["decision"], r.recompute), f"block 2 step {s}"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"block 2 step {s}")
    assert B.device_status() == 0
    return ref2


def test_gqa_batch_two_blocks():
    """Three sequences of the long-context GQA shape (H_q 32 / H_kv 8, block 64 with
    32 active rows), prefix 300: block 2 recomputes at its first step over 364 keys
    per sequence, then reuses."""
    w1 = W.long_context_gqa(steps=3, prefix=300, batch=3)
    ref2 = _two_blocks(w1, W.next_block(w1, seed=21, steps=3))
    assert ref2[0].recompute.all() and not any(r.recompute.any() for r in ref2[1:])


def test_dllm_layer_two_blocks_in_place():
    """One sequence of the 8B-dLLM layer shape (prefix 1024, block 32, tau = 4): the
    block is appended in place after the prefix."""
    w1 = W.dllm_layer(steps=4, prefix=1024)
    ref2 = _two_blocks(w1, W.next_block(w1, seed=22, steps=4, redraws=2), in_place=True)
    assert ref2[0].recompute.all() and not ref2[1].recompute.any()


def test_varlen_branches_two_blocks():
    """Six branches (blocks 4 to 128, prefix 256 each): every branch's prefix grows by
    its own block."""
    w1 = W.varlen_branches(steps=3, prefix=256)
    _two_blocks(w1, W.next_block(w1, seed=23, steps=3, redraws=3))
