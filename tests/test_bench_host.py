"""bench.py's multi-rank host logic on CPU with gloo (world size 2): each rank
serves its own request (distinct seeds, same shapes) and the reported time is
the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, r, _ = bench.dist_setup()
    seed = bench.shard_seed(1001, r)
    t = bench.max_over_ranks(10.0 + r, w)
    bench.barrier(w)
    wl = bench.make_workload("tiny", seed)
    q.put((r, seed, t, wl.problem.total_q, int(wl.k_out[0, 0, 0])))
    dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, s0, t0, n0, k0), (r1, s1, t1, n1, k1) = res
    assert s0 != s1                       # distinct requests per rank
    assert n0 == n1                       # same shapes (weak scaling)
    assert t0 == t1 == 11.0               # max over ranks


def test_step_bytes_dllm_layer():
    import bench
    from cached_split_attention_b200 import workloads as W
    p = W.dllm_layer(steps=1).problem
    reuse = bench.step_bytes(p, 0.0)["total"]
    dense = bench.step_bytes(p, 1.0)["total"]
    # Q 256 KiB + block K/V 512 KiB + A_full bf16 256 KiB + L 4 KiB + cache 516 KiB
    assert reuse == 262144 + 524288 + 266240 + 528384
    assert dense == reuse + 67108864


def test_extension_row_byte_models():
    """Byte models of the extension rows, counted by hand from the tensors."""
    import bench
    from cached_split_attention_b200 import workloads as W
    p = W.varlen_branches(steps=1, prefix=64).problem
    # 64 positions x 32 heads x (A_out 512 B + L_out 4 B), read and written, + valid and count
    assert bench.cache_copy_bytes(p, 5, 4, with_q_ref=False) == 2 * 64 * 32 * 516 + 2 * 32 * 5
    assert bench.cache_copy_bytes(p, 5, 4, with_q_ref=True) == 2 * 64 * 32 * 772 + 2 * 32 * 5
    assert bench.cache_copy_bytes(p, 0, 5, with_q_ref=False) == 2 * 4 * 32 * 516 + 2 * 32 * 5
    q = W.long_context_gqa(steps=1, batch=2, prefix=1000, heads_q=8, heads_kv=2).problem
    # (128 block + 10 selected rows) x 2 heads x 128 x bf16 x (K, V), read and written,
    # + the skip mask (2000 prefix tokens: 63 words) + indices
    assert bench.sparse_layout_bytes(q, 10) == 2 * 138 * 2 * 128 * 2 * 2 + 4 * 63 + 4 * (10 + 9)


def test_sparse_selection_shape():
    import bench
    sel = bench.sparse_selection([32768, 1061])
    for s, n in zip(sel, [32768, 1061]):
        assert len(s) == 64 + 32 + 256 and np.all(np.diff(s) > 0) and s[0] == 0 and s[-1] == n - 1
        assert np.array_equal(s[:64], np.arange(64)) and np.array_equal(s[-256:], np.arange(n - 256, n))


def test_cpu_baseline_reports_its_host():
    """The oracle baseline states the threads it used, nproc and the CPU model."""
    import bench
    out = bench.cpu_baseline("tiny", 1000, budget_s=0.05)
    assert out["kind"] == "oracle" and out["value"] > 0 and out["cores"] >= 1
    assert out["host"]["nproc"] == os.cpu_count()
    assert out["host"]["cpu_model"] is None or isinstance(out["host"]["cpu_model"], str)


def test_oracle_sample_of_the_gqa_batch_is_its_first_sequence():
    """The CPU legs time one of the long-context batch's equal sequences and scale by
    the batch size: the sample must be exactly sequence 0 of the batch (same rows,
    keys and decisions as in the whole batch)."""
    from cached_split_attention_b200 import workloads as W
    from oracle import policy
    w = W.long_context_gqa(steps=3, prefix=96, batch=3)
    one = W.first_sequences(w, 1)
    assert one.problem.num_seqs == 1 and one.problem.total_kv_out == 96
    full = policy.run_policy(w)
    part = policy.run_policy(one)
    for f, p in zip(full, part):
        n = p.problem.total_q
        assert np.array_equal(f.recompute[:1], p.recompute)
        assert np.array_equal(f.a_full[:n], p.a_full) and np.array_equal(f.l_full[:n], p.l_full)
