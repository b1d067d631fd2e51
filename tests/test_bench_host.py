"""bench.py's multi-rank host logic on CPU with gloo (world size 2): each rank
serves its own request (distinct seeds, same shapes) and the reported time is
the maximum over ranks."""
import os
import socket

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
