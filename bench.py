"""Benchmark of the FlashBlock denoise-step attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload long_context_gqa|dllm_layer|varlen_branches|video|tiny]
                    [--layers L] [--headline-only] [--rows]

The headline workload (default: long-context GQA, the largest configuration:
batch 8, prefix 32768, 1 GiB of prefix K/V per layer) gives the JSON line; on one
GPU the other four configurations are then timed the same way and carried under
"configs" of that line (--headline-only skips them).

The workload is run the way a block-diffusion model runs it: every denoise step
calls the attention of each of L layers (32 for the 8B dLLM), and every layer has
its own prefix K/V, FlashBlock cache and block inputs (distinct device buffers;
the prefixes alone are L x 64 MiB = 2 GiB for the 8B-dLLM layer, far above L2).
L2 is flushed (a 256 MiB read, untimed) before every denoise step, so each call
starts with its data cold.  The L calls of a denoise step are replayed as one CUDA
graph and timed with CUDA events on the launching stream.

One bench step is one denoise episode of the block: the caches are invalidated
(untimed set-up of a new block), step 0 recomputes, later steps follow the workload's reuse gates (32 denoise
steps x L layers = 1024 fb_step calls for the 8B-dLLM layer).  `value` is the
mean latency of one attention call (one layer, one denoise step) in microseconds
over the K timed episodes (max over ranks).

`e2e` is the same metric through the public API with host buffers: each denoise
step's graph also copies every layer's block Q/K/V and update count from pinned
host memory and copies A_full and L_full back, on two copy streams that overlap
the uploads and downloads with the other layers' attention.

`roofline` is the attention kernel that serves the workload (KERNEL_OF) on its
recompute launches (prefix pass + block pass + merge): HBM-bound workloads report
algorithmic bytes per launch / launch time against the measured copy bandwidth,
the video block (a dense contraction) algorithmic flops / time against the
measured sustained bf16 tensor throughput; `roofline_all_launches` aggregates
every launch.

`--impl reference` times the fp64 oracle (the plain CPU statement of the method)
on the host cores on one layer of the same workload, rank 0 only (for the
long-context GQA batch: one of its 8 equal sequences, the time scaled by 8).

`--rows` measures the extension rows instead (one JSON line, one GPU): the
cumulative-M gate on the 8B-dLLM layer, the BlockBatch branch hooks on the
varlen-branch problem, and the sparse-residual layout and step on the
long-context GQA problem (see `rows`).

With torchrun (N > 1) every rank runs its own request (seed + rank) on its own
GPU with no collective on the data path (weak scaling); ranks meet only at the
barriers around the timed region and in the max-reduction of the timings.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from cached_split_attention_b200 import workloads as W  # noqa: E402

METRIC = "denoise-step attention µs; effective KV TB/s vs ~8 TB/s HBM peak"
WORKLOAD_DESC = {
    "dllm_layer": "8B-dLLM layer: batch 1, bf16 MHA H=32, d=128, prefix 4096, block 32, 32 steps, "
                  "1-4 redraws/step (Poisson mean 2), tau=4",
    "long_context_gqa": "long context GQA: batch 8, H_q=32, H_kv=8, d=128, prefix 32768, block 64, "
                        "16 steps, 50% rows locked, forced reuse after step 0",
    "varlen_branches": "varlen branches: 6 branches B=4..128, prefix 2048 each, H=32, d=128, 8 steps, tau=4",
    "video": "video-shaped: H=40, d=128, block 1560, prefix 9360, 10 steps, gamma=0.95",
    "tiny": "tiny: H=4, d=64, prefix 256, block 32, 4 steps, tau=8",
}


# ---------------------------------------------------------------- algorithmic bytes

def step_bytes(p, recompute_heads_frac: float) -> dict:
    """Bytes the method must move in one denoise step (counted from the tensors):
    Q rows + K/V of the block + A_full (bf16) and L_full, plus for heads that
    recompute the prefix K/V and the cache write (A_out fp32 + L_out), and for
    heads that reuse the cache read."""
    H, Hk, d = p.num_heads_q, p.num_heads_kv, p.head_dim
    q = p.total_q * H * d * 2
    kv_in = p.total_kv_in * Hk * d * 2 * 2
    out = p.total_q * H * (d * 2 + 4)
    cache = p.total_q * H * (d * 4 + 4)
    kv_out = p.total_kv_out * Hk * d * 2 * 2
    f = recompute_heads_frac
    return dict(total=q + kv_in + out + f * (kv_out + cache) + (1 - f) * cache,
                kv_out=f * kv_out)


def step_flops(p, recompute_heads_frac: float) -> float:
    H, d = p.num_heads_q, p.head_dim
    lens_q = np.diff(p.cu_seqlens_q).astype(np.float64)
    lens_o = np.diff(p.cu_seqlens_kv_out).astype(np.float64)
    lens_i = np.diff(p.cu_seqlens_kv_in).astype(np.float64)
    return float(4 * H * d * (np.sum(lens_q * lens_i) + recompute_heads_frac * np.sum(lens_q * lens_o)))


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self.period = period_s
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        reasons = [name for bit, name in self.REASONS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ---------------------------------------------------------------- distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank serves its own request: a different seed, same shapes."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def make_workload(name: str, seed: int):
    fn = W.NAMED[name]
    return fn(seed=seed)


# ---------------------------------------------------------------- native arm

DEFAULT_LAYERS = {"dllm_layer": 32, "long_context_gqa": 32, "varlen_branches": 32, "video": 8, "tiny": 32}


class Model:
    """L layers of one workload shape on the device, run through fb_step.

    Layer l holds its own copies of the prefix K/V, the block inputs of every
    step, the FlashBlock cache, the workspace and the outputs."""

    def __init__(self, w, layers, device):
        import torch
        from cached_split_attention_b200 import binding as B
        self.torch, self.B, self.w, self.L = torch, B, w, layers
        S = len(w.steps)
        self.S = S
        p = w.problem
        self.dp = [B.DeviceProblem(st.problem, device) for st in w.steps]
        wsz = max(B.workspace_size(d) for d in self.dp)
        k_out0, v_out0 = B.bf16_tensor(w.k_out, device), B.bf16_tensor(w.v_out, device)
        H, d = p.num_heads_q, p.head_dim
        tq = max(st.problem.total_q for st in w.steps)
        # Each step's block inputs of a layer live in one device blob (Q, K_in, V_in,
        # n_updated at 256-byte aligned offsets) and the outputs in another (A_full,
        # L_full), so the end-to-end leg moves each with a single copy; the pinned
        # host blobs have the same layout (the inputs are shared by the layers).
        self.in_layout = []
        host_in = []
        for st in w.steps:
            parts = [st.q.view(np.uint8).reshape(-1), st.k_in.view(np.uint8).reshape(-1),
                     st.v_in.view(np.uint8).reshape(-1), st.n_updated.astype(np.int32).view(np.uint8)]
            offs, off = [], 0
            for a in parts:
                offs.append(off)
                off = (off + a.nbytes + 255) // 256 * 256
            blob = np.zeros(off, dtype=np.uint8)
            for o, a in zip(offs, parts):
                blob[o:o + a.nbytes] = a
            self.in_layout.append((offs, [a.nbytes for a in parts], st.q.shape, st.k_in.shape))
            host_in.append(blob)
        a_bytes = (tq * H * d * 2 + 255) // 256 * 256
        self.out_bytes = a_bytes + tq * H * 4
        self.layers = []
        for _ in range(layers):
            lay = dict(k_out=k_out0.clone(), v_out=v_out0.clone(), inb=[], q=[], k_in=[], v_in=[], n=[],
                       cache=B.Cache(p, device, with_q_ref=bool(w.flags & W.GATE_HEAD)),
                       ws=torch.empty(wsz, dtype=torch.uint8, device=device),
                       outb=torch.empty(self.out_bytes, dtype=torch.uint8, device=device),
                       dec=torch.empty((p.num_seqs, H), dtype=torch.uint8, device=device))
            for s_, blob in enumerate(host_in):
                offs, sizes, qshape, kshape = self.in_layout[s_]
                dblob = torch.from_numpy(blob).to(device)
                lay["inb"].append(dblob)
                lay["q"].append(dblob[offs[0]:offs[0] + sizes[0]].view(torch.bfloat16).view(qshape))
                lay["k_in"].append(dblob[offs[1]:offs[1] + sizes[1]].view(torch.bfloat16).view(kshape))
                lay["v_in"].append(dblob[offs[2]:offs[2] + sizes[2]].view(torch.bfloat16).view(kshape))
                lay["n"].append(dblob[offs[3]:offs[3] + sizes[3]].view(torch.int32))
            lay["a_full"] = lay["outb"][:tq * H * d * 2].view(torch.bfloat16).view(tq, H, d)
            lay["l_full"] = lay["outb"][a_bytes:a_bytes + tq * H * 4].view(torch.float32).view(tq, H)
            B.workspace_init(lay["ws"])
            self.layers.append(lay)
        del k_out0, v_out0
        self.h_in = [torch.from_numpy(b).pin_memory() for b in host_in]
        self.h_out = [torch.empty(self.out_bytes, dtype=torch.uint8).pin_memory() for _ in range(layers)]
        # L2 flush: read 256 MiB (about twice the L2)
        self.flush_buf = torch.ones(64 << 20, dtype=torch.int32, device=device)
        self.flush_out = torch.empty((), dtype=torch.int32, device=device)
        self.graphs = {}
        # end-to-end leg: inputs come in on one copy stream, results leave on
        # another, so layer l+1's upload and layer l-1's download overlap layer l
        self.copy_in = torch.cuda.Stream(device)
        self.copy_out = torch.cuda.Stream(device)
        self.ev_in = [torch.cuda.Event() for _ in range(layers)]
        self.ev_done = [torch.cuda.Event() for _ in range(layers)]

    def call(self, li, s, prm, stream):
        lay = self.layers[li]
        self.B.step(self.dp[s], prm, lay["cache"], lay["q"][s], lay["k_in"][s], lay["v_in"][s], lay["k_out"],
                    lay["v_out"], lay["n"][s], lay["a_full"], lay["ws"], l_full=lay["l_full"], decision_out=lay["dec"],
                    stream=stream)

    def denoise_step(self, s, prm, stream, e2e=False):
        """Attention of every layer for denoise step s."""
        if e2e:
            return self.denoise_step_e2e(s, prm, stream)
        for li in range(self.L):
            self.call(li, s, prm, stream)

    def denoise_step_e2e(self, s, prm, stream):
        """The same with host buffers: each layer's block Q/K/V and update count are
        uploaded from pinned memory and its A_full / L_full read back, the copies on
        their own streams so that they overlap the other layers' attention."""
        torch, B = self.torch, self.B
        self.copy_in.wait_stream(stream)
        self.copy_out.wait_stream(stream)
        for li in range(self.L):
            lay = self.layers[li]
            with torch.cuda.stream(self.copy_in):
                lay["inb"][s].copy_(self.h_in[s], non_blocking=True)  # Q, K_in, V_in, n_updated
                self.ev_in[li].record(self.copy_in)
            stream.wait_event(self.ev_in[li])
            B.step(self.dp[s], prm, lay["cache"], lay["q"][s], lay["k_in"][s], lay["v_in"][s], lay["k_out"],
                   lay["v_out"], lay["n"][s], lay["a_full"], lay["ws"], l_full=lay["l_full"], decision_out=lay["dec"],
                   stream=stream)
            self.ev_done[li].record(stream)
            self.copy_out.wait_event(self.ev_done[li])
            with torch.cuda.stream(self.copy_out):
                self.h_out[li].copy_(lay["outb"], non_blocking=True)  # A_full, L_full
        stream.wait_stream(self.copy_in)
        stream.wait_stream(self.copy_out)

    def new_block(self, stream):
        """A new block starts: every layer's cache is empty (episode set-up, untimed)."""
        for lay in self.layers:
            self.B.cache_invalidate(self.dp[0], lay["cache"], stream=stream)

    def graph(self, s, flags, e2e):
        key = (s, flags, e2e)
        if key not in self.graphs:
            torch = self.torch
            prm = self.B.params(self.w.tau, self.w.gamma, flags)
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                self.denoise_step(s, prm, side, e2e)  # warm-up outside capture
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.denoise_step(s, prm, torch.cuda.current_stream(), e2e)
            torch.cuda.synchronize()
            self.graphs[key] = (g, prm)
        return self.graphs[key][0]

    def episode(self, flags, events=None, e2e=False):
        torch = self.torch
        stream = torch.cuda.current_stream()
        for s in range(self.S):
            g = self.graph(s, flags, e2e)
            if s == 0:
                self.new_block(stream)
            torch.amax(self.flush_buf, dim=0, out=self.flush_out)
            if events is not None:
                events[s][0].record(stream)
            g.replay()
            if events is not None:
                events[s][1].record(stream)

    def e2e_bytes(self, s):
        """Bytes of the two copies of one call (the blobs, alignment padding included)."""
        return int(self.h_in[s].numel()), int(self.out_bytes)


def _events(torch, K, S):
    return [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(S)]
            for _ in range(K)]


def _elapsed_us(ev):
    return np.array([[e0.elapsed_time(e1) * 1e3 for e0, e1 in row] for row in ev])


# The attention kernel that serves each workload's fused step (planned by
# fb_api.cu: head_dim 128 with more than 64 rows per group -> tensor-core kernel,
# multi-head with 256+ rows per head -> its two-tile form) and the sources it is
# built from.
KERNEL_OF = {"dllm_layer": "attn_kernel", "tiny": "attn_kernel", "long_context_gqa": "tc_attn_kernel",
             "varlen_branches": "tc_attn_kernel", "video": "tc2_attn_kernel"}
_BASE_SOURCES = ("fb_device.cuh", "fb_kernels.cuh", "fb_reuse.cuh")
KERNEL_SOURCES = {"attn_kernel": _BASE_SOURCES,
                  "tc_attn_kernel": _BASE_SOURCES + ("fb_tcgen05.cuh", "fb_tc_kernel.cuh"),
                  "tc2_attn_kernel": _BASE_SOURCES + ("fb_tcgen05.cuh", "fb_tc_kernel.cuh", "fb_tc2_kernel.cuh")}


def kernel_source_digest(kernel: str = "attn_kernel") -> str:
    """sha256 over the device sources of one attention kernel (its code and device
    helpers); the DRAM counters recorded for it in profiles/traffic.json are
    reported only while this digest matches."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "cached_split_attention_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


SEED_OF = {"tiny": 1000, "dllm_layer": 1001, "long_context_gqa": 1002, "varlen_branches": 1003, "video": 1004}
# The configurations measured after the headline one in a default run (one GPU):
# each gets its own line under "configs" of the same JSON object.
EXTRA_ORDER = ("dllm_layer", "varlen_branches", "video", "tiny")


def measure(name, args, world, rank, local, device):
    """Time one workload as a model runs it (see the module docstring); returns the
    JSON object of its line on rank 0 (None elsewhere)."""
    import torch
    base = SEED_OF[name]
    w = make_workload(name, shard_seed(base, rank))
    L = (args.layers if name == args.workload else 0) or DEFAULT_LAYERS[name]
    model = Model(w, L, device)
    S = model.S
    p = w.problem

    # decisions of the episode (identical for every layer): one eager pass
    stream = torch.cuda.current_stream()
    prm = model.B.params(w.tau, w.gamma, w.flags)
    lay0 = model.layers[0]
    model.B.cache_invalidate(model.dp[0], lay0["cache"], stream=stream)
    rec_frac = []
    for s in range(S):
        model.call(0, s, prm, stream)
        rec_frac.append(float(lay0["dec"].float().mean().item()))

    for _ in range(args.warmup):
        model.episode(w.flags)
    torch.cuda.synchronize()

    ev = _events(torch, args.steps, S)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for k in range(args.steps):
            model.episode(w.flags, events=ev[k])
        torch.cuda.synchronize()
    barrier(world)
    step_us = _elapsed_us(ev)                       # [K, S]: L calls each
    call_us = float(step_us.mean() / L)
    episode_ms = float(step_us.sum(axis=1).mean() * 1e-3)

    # end-to-end leg: host buffers, copies inside every step's graph
    ev2 = _events(torch, args.steps, S)
    model.episode(w.flags, e2e=True)
    torch.cuda.synchronize()
    barrier(world)
    for k in range(args.steps):
        model.episode(w.flags, events=ev2[k], e2e=True)
    torch.cuda.synchronize()
    barrier(world)
    e2e_call_us = float(_elapsed_us(ev2).mean() / L)
    h2d = sum(model.e2e_bytes(s)[0] for s in range(S)) / S
    d2h = sum(model.e2e_bytes(s)[1] for s in range(S)) / S

    # dense (forced recompute) and reuse (forced reuse) calls
    reps = max(3, min(args.steps, 10))
    evd, evr = _events(torch, reps, S), _events(torch, reps, S)
    model.episode(W.FORCE_RECOMPUTE)
    model.episode(W.FORCE_REUSE)
    for k in range(reps):
        model.episode(W.FORCE_RECOMPUTE, events=evd[k])
    for k in range(reps):
        model.episode(W.FORCE_REUSE, events=evr[k])
    torch.cuda.synchronize()
    dense_us = _elapsed_us(evd) / L
    reuse_us = _elapsed_us(evr)[:, 1:] / L

    # roofline of the fused kernel on the recompute steps of the timed episodes
    rec_steps = [s for s in range(S) if rec_frac[s] > 0]
    bytes_rec = [step_bytes(w.steps[s].problem, rec_frac[s])["total"] for s in rec_steps]
    t_rec = step_us[:, rec_steps].mean(axis=0) / L * 1e-6 if rec_steps else np.array([np.nan])
    ach_rec = float(np.sum(bytes_rec) / np.sum(t_rec) / 1e9) if rec_steps else float("nan")
    bytes_all = sum(step_bytes(w.steps[s].problem, rec_frac[s])["total"] for s in range(S))
    ach_all = bytes_all / (episode_ms * 1e-3 / L) / 1e9
    peaks = _peaks()
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    kernel = KERNEL_OF[name]
    traffic = traffic_alg = None
    try:
        prof = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        for ent in prof.get("entries", []):
            # counters only count for the kernel source they were taken on
            if (ent.get("workload") == name and ent.get("kernel") == kernel
                    and ent.get("kernel_source_sha256") == kernel_source_digest(kernel)):
                traffic = ent.get("dram_bytes_per_recompute_launch")
                traffic_alg = ent.get("algorithmic_bytes_of_that_launch")
    except Exception:
        pass
    # the video block is a dense contraction (about 1500 flop per byte): its bound
    # is the tensor cores, timed inside a long step (the sustained bf16 figure)
    tensor_bound = name == "video"
    flops_rec = [step_flops(w.steps[s].problem, rec_frac[s]) for s in rec_steps]
    ach_tf = float(np.sum(flops_rec) / np.sum(t_rec) / 1e12) if rec_steps else float("nan")
    tf_peak = float(peaks.get("bf16_tflops_sustained", 1400.0))
    tf_src = "measured, sustained" if "bf16_tflops_sustained" in peaks else "fallback, sustained"

    value = max_over_ranks(call_us, world, device)
    e2e_v = max_over_ranks(e2e_call_us, world, device)
    ms_step = max_over_ranks(episode_ms, world, device)
    clocks = sampler.summary()
    del model
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    dense_b = step_bytes(p, 1.0)["total"]
    reuse_b = step_bytes(p, 0.0)["total"]
    dense_med = float(np.median(dense_us))
    reuse_med = float(np.median(reuse_us))
    n_launch = args.steps * L * sum(launches_per_call(w, s) for s in range(S))
    return {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "us/attention-call (one layer, one denoise step)",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": WORKLOAD_DESC[name],
            "layers": L,
            "bench_step": f"one denoise episode: {S} denoise steps x {L} layers = {S * L} fb_step calls",
            "recompute_steps_per_episode": len(rec_steps),
            "l2": "flushed before every denoise step (256 MiB read, untimed); each layer's data is distinct",
            "launch": "each denoise step's L calls replayed as one CUDA graph",
            "parallelism": f"replicas x{world} (one request per GPU, no collective)",
            "seed": shard_seed(base, rank),
        },
        "throughput": {"attention_calls_per_s_all_gpus": round(world * 1e6 / value, 1)},
        "dense_call_us": {"median": round(dense_med, 3), "p10": round(float(np.percentile(dense_us, 10)), 3),
                          "p90": round(float(np.percentile(dense_us, 90)), 3),
                          "effective_tbps": round(dense_b / dense_med / 1e6, 3),
                          "frac_of_hbm": round(dense_b / dense_med / 1e3 / hbm_peak, 4),
                          "tflops": round(step_flops(p, 1.0) / dense_med / 1e6, 1)},
        "reuse_call_us": {"median": round(reuse_med, 3), "p10": round(float(np.percentile(reuse_us, 10)), 3),
                          "p90": round(float(np.percentile(reuse_us, 90)), 3),
                          "effective_tbps": round(reuse_b / reuse_med / 1e6, 3),
                          "frac_of_hbm": round(reuse_b / reuse_med / 1e3 / hbm_peak, 4)},
        "reuse_gain": {"predicted_bytes_ratio": round(dense_b / reuse_b, 2),
                       "achieved_time_ratio": round(dense_med / reuse_med, 2)},
        "roofline": dict(
            ({"bound": "tensor", "achieved": round(ach_tf, 1), "peak": tf_peak, "unit": "TFLOP/s",
              "frac": round(ach_tf / tf_peak, 4), "peak_source": tf_src, "hbm_gbs_achieved": round(ach_rec, 1)}
             if tensor_bound else
             {"bound": "hbm", "achieved": round(ach_rec, 1), "peak": hbm_peak, "unit": "GB/s",
              "frac": round(ach_rec / hbm_peak, 4), "peak_source": peak_src}),
            kernel=f"{kernel}, recompute launches (prefix + block pass + merge)", traffic=traffic,
            # the captured launch recomputes every head; the episode's recompute
            # launches may recompute fewer (gated heads), so compare with this
            traffic_launch_algorithmic_bytes=traffic_alg,
            algorithmic_bytes_per_launch=round(float(np.mean(bytes_rec))) if rec_steps else None,
            algorithmic_flops_per_launch=round(float(np.mean(flops_rec))) if rec_steps else None,
            launches=len(rec_steps) * L * args.steps),
        "roofline_all_launches": {"achieved": round(ach_all, 1), "unit": "GB/s",
                                  "frac": round(ach_all / hbm_peak, 4),
                                  "algorithmic_bytes_per_episode_per_layer": round(bytes_all)},
        "e2e": {"value": round(e2e_v, 3), "unit": "us/attention-call (one layer, one denoise step)",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "note": "bytes per attention call; each denoise step moves L times this"},
        "gpu_launches": int(n_launch),
        "clocks": clocks,
    }


def launches_per_call(w, s: int) -> int:
    """Kernels one fb_step call of step s launches: the attention kernel; the
    similarity kernel under the gamma gate; the work-order pass when the two-tile
    kernel runs with the gates on (from the library's own plan)."""
    from cached_split_attention_b200 import binding as B
    p = w.steps[s].problem
    gated = not (w.flags & (W.FORCE_RECOMPUTE | W.FORCE_REUSE))
    plan = B.plan_query(B.DeviceProblem(p, "cpu"), B.CALL_STEP)
    two_tile = plan["kernel_name"] == "tc2_attn_kernel"
    return 1 + (1 if gated and w.flags & W.GATE_HEAD else 0) + (1 if gated and two_tile else 0)


def config_summary(line: dict) -> dict:
    """The keys of a configuration's line carried under "configs" of the headline."""
    keys = ("value", "unit", "ms_per_step", "dense_call_us", "reuse_call_us", "reuse_gain", "roofline", "e2e",
            "gpu_launches", "clocks")
    out = {k: line[k] for k in keys}
    out["config"] = {k: line["config"][k] for k in ("workload", "layers", "bench_step", "recompute_steps_per_episode",
                                                    "seed")}
    return out


def native(args, world, rank, local):
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    out = measure(args.workload, args, world, rank, local, device)
    # the other configurations, one GPU only (their lines ride along under "configs")
    extra = [n for n in EXTRA_ORDER if n != args.workload] if (world == 1 and not args.headline_only) else []
    if extra and rank == 0:
        out["configs"] = {}
        for name in extra:
            out["configs"][name] = config_summary(measure(name, args, world, rank, local, device))
    if rank != 0:
        _teardown(world)
        return
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, shard_seed(SEED_OF[args.workload], rank),
                                           budget_s=args.cpu_budget)
    print(json.dumps(out), flush=True)
    _teardown(world)


# ---------------------------------------------------------------- extension rows

def sparse_selection(prefix_lens, seed: int = 7, sink: int = 64, window: int = 256, middle: int = 32):
    """A static sparse pattern per sequence: the first `sink` prefix keys, the last
    `window`, and `middle` seeded keys in between (increasing positions)."""
    rng = np.random.default_rng(seed)
    out = []
    for n in prefix_lens:
        n = int(n)
        mid = rng.choice(np.arange(sink, n - window), size=middle, replace=False)
        out.append(np.unique(np.concatenate([np.arange(sink), mid, np.arange(n - window, n)])).astype(np.int32))
    return out


def sparse_layout_bytes(p, total_sel: int) -> int:
    """Bytes fb_sparse_layout must move: the block rows and the selected prefix rows
    (K and V) read once and written once into J_in', the prefix skip mask written, and
    the index arrays read."""
    row = p.num_heads_kv * p.head_dim * 2 * 2          # K and V, bf16
    mask = 4 * ((p.total_kv_out + 31) // 32)
    return 2 * (p.total_kv_in + total_sel) * row + mask + 4 * (total_sel + 3 * (p.num_seqs + 1))


def cache_copy_bytes(p, src: int, dst: int, with_q_ref: bool) -> int:
    """Bytes fb_cache_copy_seq must move: the entries of min(B_src, B_dst) block
    positions (A_out fp32, L_out, and q_ref bf16 when the cache has it), read and
    written, plus the per-head valid flags and update counts."""
    n = min(int(p.lens("in")[src]), int(p.lens("in")[dst]))
    per = p.num_heads_q * (p.head_dim * 4 + 4 + (p.head_dim * 2 if with_q_ref else 0))
    return 2 * n * per + 2 * p.num_heads_q * 5


def _graph_of(torch, fn):
    """fn(stream) captured as a CUDA graph (run once eagerly first, outside capture)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


def _cold_us(torch, g, flush, flush_out, reps: int, clocks: "ClockSampler") -> np.ndarray:
    """Device time of one replay of graph g, each after an untimed 256 MiB read that
    evicts L2; CUDA events on the launching stream; µs per replay.  The SM clock
    samples taken meanwhile are added to `clocks`."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    g.replay()
    torch.cuda.synchronize()
    with ClockSampler(clocks.index) as cs:
        for e0, e1 in ev:
            torch.amax(flush, dim=0, out=flush_out)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    clocks.samples += cs.samples
    return np.array([e0.elapsed_time(e1) * 1e3 for e0, e1 in ev])


def _stats(t: np.ndarray) -> dict:
    return {"median": round(float(np.median(t)), 3), "p10": round(float(np.percentile(t, 10)), 3),
            "p90": round(float(np.percentile(t, 90)), 3)}


def _peaks() -> dict:
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {}


class _Single:
    """One layer of one step of a problem on the device: inputs, cache, workspace,
    outputs (the shapes fb_step wants)."""

    def __init__(self, B, torch, problem, st, k_out, v_out, device, with_q_ref=False, kv_out_skip=None):
        self.B, self.dp = B, B.DeviceProblem(problem, device, kv_out_skip=kv_out_skip)
        H, d = problem.num_heads_q, problem.head_dim
        self.q = B.bf16_tensor(st.q, device)
        self.k_in, self.v_in = B.bf16_tensor(st.k_in, device), B.bf16_tensor(st.v_in, device)
        self.k_out, self.v_out = k_out, v_out
        self.n = torch.as_tensor(st.n_updated.astype(np.int32)).to(device)
        self.cache = B.Cache(problem, device, with_q_ref=with_q_ref)
        self.ws = torch.empty(B.workspace_size(self.dp), dtype=torch.uint8, device=device)
        B.workspace_init(self.ws)
        self.a = torch.empty((max(problem.total_q, 1), H, d), dtype=torch.bfloat16, device=device)
        self.l = torch.empty((max(problem.total_q, 1), H), dtype=torch.float32, device=device)

    def step(self, prm, stream):
        self.B.step(self.dp, prm, self.cache, self.q, self.k_in, self.v_in, self.k_out, self.v_out, self.n, self.a,
                    self.ws, l_full=self.l, stream=stream)


def rows(args, world, rank, local):
    """Measurements of the extension rows on one GPU, one JSON line (rank 0 only):

    * cumulative-M gate: the 8B-dLLM layer's episodes (L layers, graphs, L2 flushed
      before every denoise step, as the headline) under FB_GATE_TAU_CUM, beside the
      per-step gate on the same model;
    * BlockBatch hooks on the varlen-branch problem: leader sync (fb_cache_copy_seq,
      the 128-token branch's entries to the 64-token branch) and refresh
      (fb_cache_invalidate_seqs of one branch), each after an L2 flush;
    * sparse residual on the long-context GQA problem (8 x 32768 prefix): the layout
      pass (fb_sparse_layout) and fb_step on the laid-out keys (forced recompute and
      forced reuse), beside fb_step on the dense keys, each after an L2 flush."""
    if rank != 0:
        return
    import torch
    from cached_split_attention_b200 import binding as B
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    flush = torch.ones(64 << 20, dtype=torch.int32, device=device)
    flush_out = torch.empty((), dtype=torch.int32, device=device)
    peaks = _peaks()
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    reps = max(10, min(args.steps, 50))
    out_rows, launches = {}, 0
    clocks = ClockSampler(local)        # collects the samples of every timed region
    stream = torch.cuda.current_stream()
    if args.rows in ("all", "gate"):
        launches += _rows_gate(args, torch, B, device, local, clocks, out_rows, hbm_peak, peak_src)
    if args.rows in ("all", "hooks"):
        launches += _rows_hooks(torch, B, device, stream, flush, flush_out, reps, clocks, out_rows, hbm_peak,
                                peak_src)
    if args.rows in ("all", "sparse"):
        launches += _rows_sparse(torch, B, device, flush, flush_out, reps, clocks, out_rows, hbm_peak, peak_src)
    if B.device_status() != 0:
        raise RuntimeError("device status set during the extension-row measurements")
    out = {"metric": "extension rows: device µs per call", "impl": "native", "bench": "rows", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "dtype": "bf16", "data": "synthetic",
           "l2": "flushed (256 MiB read, untimed) before every timed denoise step or call",
           "rows": out_rows, "gpu_launches": int(launches), "clocks": clocks.summary()}
    print(json.dumps(out), flush=True)


def _rows_gate(args, torch, B, device, local, clocks, out_rows, hbm_peak, peak_src) -> int:
    """Cumulative-M gate against the per-step gate, 8B-dLLM layer episodes."""
    launches = 0
    w = make_workload("dllm_layer", 1001)
    L = args.layers or DEFAULT_LAYERS["dllm_layer"]
    model = Model(w, L, device)
    S = model.S
    stream = torch.cuda.current_stream()
    lay0 = model.layers[0]
    gate = {}
    for name, flags in (("per_step", W.GATE_TAU), ("cumulative", W.GATE_TAU_CUM)):
        prm = B.params(w.tau, w.gamma, flags)
        B.cache_invalidate(model.dp[0], lay0["cache"], stream=stream)
        rec = []
        for s in range(S):
            model.call(0, s, prm, stream)
            rec.append(float(lay0["dec"].float().mean().item()))
        for _ in range(args.warmup):
            model.episode(flags)
        ev = _events(torch, args.steps, S)
        torch.cuda.synchronize()
        with ClockSampler(local) as cs:
            for k in range(args.steps):
                model.episode(flags, events=ev[k])
            torch.cuda.synchronize()
        clocks.samples += cs.samples
        launches += args.steps * S * L
        step_us = _elapsed_us(ev)
        rs = [s for s in range(S) if rec[s] > 0]
        t_rec = step_us[:, rs].mean(axis=0) / L * 1e-6
        b_rec = [step_bytes(w.steps[s].problem, rec[s])["total"] for s in rs]
        ach = float(np.sum(b_rec) / np.sum(t_rec) / 1e9)
        gate[name] = {"us_per_call": round(float(step_us.mean() / L), 3),
                      "recompute_steps_per_episode": len(rs),
                      "recompute_call_us": round(float(np.mean(t_rec)) * 1e6, 3),
                      "roofline": {"bound": "hbm", "kernel": "attn_kernel, recompute launches",
                                   "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                                   "frac": round(ach / hbm_peak, 4), "peak_source": peak_src}}
    out_rows["cumulative_gate"] = dict(
        workload=WORKLOAD_DESC["dllm_layer"] + f"; {L} layers, {S}-step episodes", tau=w.tau, **gate)
    del model, lay0
    torch.cuda.empty_cache()
    return launches


def _rows_hooks(torch, B, device, stream, flush, flush_out, reps, clocks, out_rows, hbm_peak, peak_src) -> int:
    """BlockBatch leader sync and refresh on the varlen-branch problem: one call
    after an L2 flush, and 32 calls back to back in one graph (per-call time)."""
    launches = 0
    w = make_workload("varlen_branches", 1003)
    p = w.problem
    one = _Single(B, torch, p, w.steps[0], B.bf16_tensor(w.k_out, device), B.bf16_tensor(w.v_out, device),
                  device)
    one.step(B.params(0, 0.0, W.FORCE_RECOMPUTE), stream)   # fill every branch's entries
    src, dst = int(np.argmax(p.lens("in"))), int(np.argsort(p.lens("in"))[-2])
    mask = torch.zeros(p.num_seqs, dtype=torch.uint8, device=device)
    mask[int(np.argmin(p.lens("in")))] = 1
    copy = lambda st: B.cache_copy_seq(one.dp, one.cache, src, dst, stream=st)
    inv = lambda st: B.cache_invalidate_seqs(one.dp, one.cache, mask, stream=st)
    t_copy = _cold_us(torch, _graph_of(torch, copy), flush, flush_out, reps, clocks)
    t_inv = _cold_us(torch, _graph_of(torch, inv), flush, flush_out, reps, clocks)
    nb = 32
    many = lambda fn: (lambda st: [fn(st) for _ in range(nb)])
    t_copy_bb = _cold_us(torch, _graph_of(torch, many(copy)), flush, flush_out, reps, clocks) / nb
    t_inv_bb = _cold_us(torch, _graph_of(torch, many(inv)), flush, flush_out, reps, clocks) / nb
    launches += 2 * reps * (1 + nb)
    cb = cache_copy_bytes(p, src, dst, with_q_ref=False)
    ach = cb / float(np.median(t_copy)) / 1e3
    out_rows["branch_hooks"] = {
        "workload": WORKLOAD_DESC["varlen_branches"],
        "leader_sync": dict(_stats(t_copy), call="fb_cache_copy_seq", src_block=int(p.lens("in")[src]),
                            dst_block=int(p.lens("in")[dst]), algorithmic_bytes=cb,
                            roofline={"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak,
                                      "unit": "GB/s", "frac": round(ach / hbm_peak, 4),
                                      "peak_source": peak_src},
                            back_to_back_us_per_call=_stats(t_copy_bb)),
        "refresh": dict(_stats(t_inv), call="fb_cache_invalidate_seqs", branches=1,
                        back_to_back_us_per_call=_stats(t_inv_bb)),
        "timing": f"median over {reps} graph replays, each after an L2 flush; back to back: "
                  f"{nb} calls in one graph, time / {nb}",
    }
    del one
    torch.cuda.empty_cache()
    return launches


def _rows_sparse(torch, B, device, flush, flush_out, reps, clocks, out_rows, hbm_peak, peak_src) -> int:
    """Sparse residual on the long-context GQA problem: the layout pass, and fb_step
    on the laid-out keys beside fb_step on the dense keys (forced recompute / reuse)."""
    import dataclasses
    launches = 0
    w = make_workload("long_context_gqa", 1002)
    p, st = w.problem, w.steps[0]
    sel = sparse_selection(p.lens("out"))
    cu_sel = np.concatenate([[0], np.cumsum([len(s) for s in sel])]).astype(np.int32)
    total_sel = int(cu_sel[-1])
    Hk, d = p.num_heads_kv, p.head_dim
    k_out, v_out = B.bf16_tensor(w.k_out, device), B.bf16_tensor(w.v_out, device)
    dense = _Single(B, torch, p, st, k_out, v_out, device)
    k_ext = torch.empty((p.total_kv_in + total_sel, Hk, d), dtype=torch.bfloat16, device=device)
    v_ext = torch.empty_like(k_ext)
    skip = torch.empty((p.total_kv_out + 31) // 32, dtype=torch.int32, device=device)
    cu_i = torch.empty(p.num_seqs + 1, dtype=torch.int32, device=device)
    d_cu_sel = torch.as_tensor(cu_sel).to(device)
    d_sel = torch.as_tensor(np.concatenate(sel)).to(device)

    def layout(stream_):
        B.sparse_layout(dense.dp, d_cu_sel, d_sel, total_sel, k_out, v_out, dense.k_in, dense.v_in, k_ext, v_ext,
                        skip, cu_i, stream=stream_)

    g_lay = _graph_of(torch, layout)
    t_lay = _cold_us(torch, g_lay, flush, flush_out, reps, clocks)
    p2 = dataclasses.replace(p, cu_seqlens_kv_in=cu_i.cpu().numpy())
    sp = _Single(B, torch, p2, dataclasses.replace(st, problem=p2), k_out, v_out, device, kv_out_skip=skip)
    sp.k_in, sp.v_in = k_ext, v_ext
    timed = {}
    for name, obj in (("sparse", sp), ("dense", dense)):
        for arm, flags in (("recompute", W.FORCE_RECOMPUTE), ("reuse", W.FORCE_REUSE)):
            prm = B.params(0, 0.0, flags)
            g = _graph_of(torch, lambda st_, o=obj, pr=prm: o.step(pr, st_))
            timed[(name, arm)] = _cold_us(torch, g, flush, flush_out, reps, clocks)
            launches += reps
            del g
    launches += reps
    # the layout where it runs: on the stream in front of the sparse recompute call
    # that reads what it writes (the difference is its marginal cost there)
    prm_rec = B.params(0, 0.0, W.FORCE_RECOMPUTE)

    def layout_then_step(st_):
        layout(st_)
        sp.step(prm_rec, st_)

    g_both = _graph_of(torch, layout_then_step)
    t_both = _cold_us(torch, g_both, flush, flush_out, reps, clocks)
    launches += 2 * reps
    del g_both
    lb = sparse_layout_bytes(p, total_sel)
    ach = lb / float(np.median(t_lay)) / 1e3

    def arm(name, a, f):
        t = timed[(name, a)]
        b = step_bytes(p2 if name == "sparse" else p, f)["total"]
        if name == "sparse":   # the selected keys are not streamed with the prefix
            b -= f * total_sel * Hk * d * 2 * 2
        return dict(_stats(t), algorithmic_bytes=round(b), frac_of_hbm=round(b / float(np.median(t)) / 1e3 /
                                                                             hbm_peak, 4))

    out_rows["sparse_residual"] = {
        "workload": WORKLOAD_DESC["long_context_gqa"],
        "selection": f"per sequence the first 64 and last 256 prefix keys and 32 seeded keys between: "
                     f"{total_sel // p.num_seqs} of {p.max_kv_out} keys",
        "layout": dict(_stats(t_lay), call="fb_sparse_layout", algorithmic_bytes=lb,
                       roofline={"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                                 "frac": round(ach / hbm_peak, 4), "peak_source": peak_src},
                       timing="alone: one call per graph replay after an L2 flush"),
        "layout_then_recompute": dict(
            _stats(t_both), calls="fb_sparse_layout then fb_step (sparse, recompute) in one graph",
            layout_marginal_us=round(float(np.median(t_both)) - float(np.median(timed[("sparse", "recompute")])), 3),
            layout_marginal_frac_of_dense_recompute=round(
                (float(np.median(t_both)) - float(np.median(timed[("sparse", "recompute")]))) /
                float(np.median(timed[("dense", "recompute")])), 4)),
        "step_sparse": {"recompute_call_us": arm("sparse", "recompute", 1.0),
                        "reuse_call_us": arm("sparse", "reuse", 0.0)},
        "step_dense": {"recompute_call_us": arm("dense", "recompute", 1.0),
                       "reuse_call_us": arm("dense", "reuse", 0.0)},
    }
    return launches


def _teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- oracle on the host

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def host_cpu() -> dict:
    """The host the oracle runs on: logical CPUs (nproc) and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def oracle_sample(name: str, seed: int):
    """The workload the CPU oracle times and the factor that scales its time to one
    full attention call: the long-context GQA batch is 8 sequences of the same
    shape, so one of them is timed and the time multiplied by 8; the other
    workloads are timed whole."""
    w = make_workload(name, seed)
    if name == "long_context_gqa":
        n = w.problem.num_seqs
        return W.first_sequences(w, 1), float(n), f"1 of the {n} sequences (same shape), time x {n}"
    return w, 1.0, "every sequence"


def cpu_baseline(workload: str, seed: int, budget_s: float = 12.0) -> dict:
    """The fp64 oracle (as it stands) on a bounded sample: whole episodes of the
    same workload (one sequence of a batch of equal sequences, scaled) until about
    budget_s seconds have passed."""
    from oracle import policy
    w, scale, what = oracle_sample(workload, seed)
    S = len(w.steps)
    t0 = time.perf_counter()
    n = 0
    while True:
        policy.run_policy(w)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(dt / (n * S) * scale * 1e6, 1), "unit": "us/attention-call (one layer, one denoise step)",
            "cores": _oracle_threads(), "host": host_cpu(), "kind": "oracle",
            "sample": f"{n} full episode(s) of {S} denoise steps of one layer, {what}, every row and head, "
                      f"fp64 numpy"}


def reference(args, world, rank):
    if rank != 0:
        return
    from oracle import policy
    w, scale, what = oracle_sample(args.workload, shard_seed(SEED_OF[args.workload], 0))
    S = len(w.steps)
    for _ in range(args.warmup):
        policy.run_policy(w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        policy.run_policy(w)
    dt = time.perf_counter() - t0
    us = dt / (args.steps * S) * scale * 1e6
    cores = _oracle_threads()
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(us, 1),
        "unit": "us/attention-call (one layer, one denoise step)",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * scale * 1e3, 3),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC[args.workload],
                   "bench_step": f"one denoise episode ({S} steps) of one layer, fp64 oracle on host cores"},
        "cpu_baseline": {"value": round(us, 1), "unit": "us/attention-call (one layer, one denoise step)",
                         "cores": cores, "host": host_cpu(), "kind": "oracle",
                         "sample": f"{args.steps} full episode(s) of {S} denoise steps of one layer, {what}, "
                                   f"every row and head"},
        "e2e": {"value": round(us, 1), "unit": "us/attention-call (one layer, one denoise step)",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_DESC), default="long_context_gqa")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only --workload (by default one GPU also times the other four configurations)")
    ap.add_argument("--layers", type=int, default=0, help="attention layers per denoise step (0: workload default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--rows", nargs="?", const="all", default=None, choices=["all", "gate", "hooks", "sparse"],
                    help="measure the extension rows (cumulative gate, branch hooks, sparse residual) instead")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.rows and args.impl == "native":
        rows(args, world, rank, local)
    elif args.impl == "reference":
        reference(args, world, rank)
    else:
        native(args, world, rank, local)


if __name__ == "__main__":
    main()
