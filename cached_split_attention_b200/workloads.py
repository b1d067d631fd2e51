"""Seeded synthetic inputs for the denoise-step attention path.

This module only draws inputs: problem shapes, bf16 bit patterns for Q/K/V and the
per-step update schedules.  It holds none of the method's arithmetic (no attention,
no merge, no gate decision), so both the CUDA path and the fp64 oracle can consume
exactly the same inputs.

Recipe (shared by all workloads):
  * values are drawn as float32 N(0, 1) from numpy's PCG64 generator, scaled in
    float32 where a workload asks for a scale, and rounded once to bf16 with
    round-to-nearest-even; the bf16 bit patterns (uint16) are what both sides read;
  * layouts are "THD": [tokens, heads, head_dim], head_dim contiguous;
  * seeds are ``1000 + workload index`` unless a test passes its own.

The five named workloads follow the shapes the FlashBlock pages and their companion
pages describe (FlashBlock: dLLM and video block diffusion; SureLock: locked rows;
BlockBatch: varlen branches of block sizes 4..128).  Where the pages leave a
distribution open, the reading taken is written next to the generator.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

# Gate flags (same values as FB_GATE_* / FB_FORCE_* in include/flashblock.h).
GATE_TAU = 1
GATE_HEAD = 2
FORCE_RECOMPUTE = 4
FORCE_REUSE = 8
GATE_TAU_CUM = 16  # tau gate on the updated tokens summed since the last recompute


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def normal_bf16(rng: np.random.Generator, shape, scale=1.0, chunk=1 << 24) -> np.ndarray:
    """bf16 bits of scale * N(0,1), drawn in float32 in chunks (bounded host memory).

    ``scale`` may be a scalar or an array broadcastable against the trailing
    dimensions of ``shape`` (used for per-head scales)."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.uint16)
    sc = np.asarray(scale, dtype=np.float32)
    if sc.ndim == 0:
        for s0 in range(0, n, chunk):
            s1 = min(n, s0 + chunk)
            v = rng.standard_normal(s1 - s0, dtype=np.float32)
            if float(sc) != 1.0:
                v *= sc
            out[s0:s1] = f32_to_bf16_bits(v)
        return out.reshape(shape)
    # per-trailing-dims scale: draw whole leading rows so the scale broadcasts
    inner = int(np.prod(shape[1:]))
    rows_per_chunk = max(1, chunk // max(inner, 1))
    res = out.reshape(shape[0], inner)
    scb = np.broadcast_to(sc, shape[1:]).reshape(-1).astype(np.float32)
    for r0 in range(0, shape[0], rows_per_chunk):
        r1 = min(shape[0], r0 + rows_per_chunk)
        v = rng.standard_normal((r1 - r0, inner), dtype=np.float32)
        v *= scb[None, :]
        res[r0:r1] = f32_to_bf16_bits(v)
    return out.reshape(shape)


@dataclasses.dataclass
class Problem:
    """Shapes and varlen index arrays of one denoise step (host copies, int32).

    cu_seqlens_q:      [num_seqs+1] packed active query rows per sequence
    q_rows:            [total_q] block position (0..B_b-1) of each packed row
    cu_seqlens_kv_out: [num_seqs+1] prefix (out-of-block) tokens per sequence
    cu_seqlens_kv_in:  [num_seqs+1] block (in-block) tokens per sequence
    """
    num_seqs: int
    num_heads_q: int
    num_heads_kv: int
    head_dim: int
    softmax_scale: float
    cu_seqlens_q: np.ndarray
    q_rows: np.ndarray
    cu_seqlens_kv_out: np.ndarray
    cu_seqlens_kv_in: np.ndarray

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def total_kv_out(self) -> int:
        return int(self.cu_seqlens_kv_out[-1])

    @property
    def total_kv_in(self) -> int:
        return int(self.cu_seqlens_kv_in[-1])

    def lens(self, which: str) -> np.ndarray:
        cu = {"q": self.cu_seqlens_q, "out": self.cu_seqlens_kv_out, "in": self.cu_seqlens_kv_in}[which]
        return np.diff(cu)

    @property
    def max_q(self) -> int:
        return int(self.lens("q").max(initial=0))

    @property
    def max_kv_out(self) -> int:
        return int(self.lens("out").max(initial=0))

    @property
    def max_kv_in(self) -> int:
        return int(self.lens("in").max(initial=0))


@dataclasses.dataclass
class StepInput:
    """Inputs of one denoise step.

    q:         bf16 bits [total_q, H_q, d]   (active rows only, packed)
    k_in/v_in: bf16 bits [total_kv_in, H_kv, d] (every block token, locked ones too)
    n_updated: int32 [num_seqs]  block tokens whose Q/K/V changed at this step
    problem:   the step's problem (the active rows may shrink step to step)
    """
    q: np.ndarray
    k_in: np.ndarray
    v_in: np.ndarray
    n_updated: np.ndarray
    problem: Problem


@dataclasses.dataclass
class Workload:
    name: str
    problem: Problem           # problem of step 0 (shapes of the prefix and the block)
    k_out: np.ndarray          # bf16 bits [total_kv_out, H_kv, d]
    v_out: np.ndarray
    steps: List[StepInput]
    tau: int
    gamma: float
    flags: int
    notes: str = ""


def _cu(lens: Sequence[int]) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lens, dtype=np.int64))]).astype(np.int32)


def make_problem(q_rows_per_seq: Sequence[Sequence[int]], kv_out_lens, kv_in_lens,
                 num_heads_q, num_heads_kv, head_dim, softmax_scale=None) -> Problem:
    q_rows = [np.asarray(r, dtype=np.int32) for r in q_rows_per_seq]
    return Problem(
        num_seqs=len(q_rows), num_heads_q=num_heads_q, num_heads_kv=num_heads_kv,
        head_dim=head_dim,
        softmax_scale=float(softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(head_dim)),
        cu_seqlens_q=_cu([len(r) for r in q_rows]),
        q_rows=(np.concatenate(q_rows) if q_rows else np.zeros(0, np.int32)).astype(np.int32),
        cu_seqlens_kv_out=_cu(kv_out_lens),
        cu_seqlens_kv_in=_cu(kv_in_lens),
    )


def _gather_q(problem: Problem, q_block: np.ndarray) -> np.ndarray:
    """Pack the active rows of a block-position Q tensor [total_kv_in, H_q, d]."""
    idx = np.empty(problem.total_q, dtype=np.int64)
    for b in range(problem.num_seqs):
        r0, r1 = problem.cu_seqlens_q[b], problem.cu_seqlens_q[b + 1]
        idx[r0:r1] = problem.cu_seqlens_kv_in[b] + problem.q_rows[r0:r1]
    return np.ascontiguousarray(q_block[idx])


class _BlockState:
    """Per-token bf16 Q/K/V of the active blocks, with redraw and noise updates."""

    def __init__(self, rng, problem: Problem, q_scale, kv_scale, v_scale=None):
        self.rng = rng
        self.p = problem
        H, Hk, d = problem.num_heads_q, problem.num_heads_kv, problem.head_dim
        T = problem.total_kv_in
        self.q_scale = q_scale
        self.kv_scale = kv_scale
        self.v_scale = kv_scale if v_scale is None else v_scale
        self.q = normal_bf16(rng, (T, H, d), q_scale)
        self.k = normal_bf16(rng, (T, Hk, d), kv_scale)
        self.v = normal_bf16(rng, (T, Hk, d), self.v_scale)

    def redraw(self, tokens: np.ndarray):
        H, Hk, d = self.p.num_heads_q, self.p.num_heads_kv, self.p.head_dim
        n = len(tokens)
        if n == 0:
            return
        self.q[tokens] = normal_bf16(self.rng, (n, H, d), self.q_scale)
        self.k[tokens] = normal_bf16(self.rng, (n, Hk, d), self.kv_scale)
        self.v[tokens] = normal_bf16(self.rng, (n, Hk, d), self.v_scale)

    def step_input(self, n_updated, problem=None) -> StepInput:
        p = problem or self.p
        return StepInput(q=_gather_q(p, self.q), k_in=self.k.copy(), v_in=self.v.copy(),
                         n_updated=np.asarray(n_updated, dtype=np.int32), problem=p)


def _redraw_schedule(rng, problem: Problem, state: _BlockState, counts):
    """Redraw counts[b] distinct uniformly chosen block tokens of each sequence."""
    toks = []
    for b in range(problem.num_seqs):
        B = int(problem.lens("in")[b])
        k = int(min(counts[b], B))
        sel = np.sort(rng.choice(B, size=k, replace=False)) + problem.cu_seqlens_kv_in[b]
        toks.append(sel)
    state.redraw(np.concatenate(toks) if toks else np.zeros(0, np.int64))


def tiny(seed: int = 1000, sharp: float = 1.0, steps: int = 4) -> Workload:
    """batch 1, H_q=H_kv=4, d=64, prefix 256, block 32, 4 steps, tau=8.

    Q, K, V ~ N(0,1)/sqrt(d) taken literally (near-uniform attention).  ``sharp``
    multiplies Q and K only (sharp = 4*sqrt(d) gives Q, K ~ 4 N(0,1): peaked
    scores that exercise the max subtraction; V keeps its scale so outputs stay
    in the range the tolerances are stated for).  Each of steps 1..S-1 redraws 4
    distinct block tokens."""
    rng = np.random.default_rng(seed)
    B, N, H, d = 32, 256, 4, 64
    p = make_problem([np.arange(B)], [N], [B], H, H, d)
    s = sharp / math.sqrt(d)
    v = 1.0 / math.sqrt(d)
    k_out = normal_bf16(rng, (N, H, d), s)
    v_out = normal_bf16(rng, (N, H, d), v)
    st = _BlockState(rng, p, s, s, v)
    out = [st.step_input([B])]
    for _ in range(1, steps):
        _redraw_schedule(rng, p, st, [4])
        out.append(st.step_input([4]))
    return Workload("tiny", p, k_out, v_out, out, tau=8, gamma=0.0, flags=GATE_TAU,
                    notes="H4 d64 prefix256 block32; N(0,1)/sqrt(d); 4 redraws/step; tau=8")


def dllm_layer(seed: int = 1001, steps: int = 32, prefix: int = 4096, block: int = 32,
               heads: int = 32, head_dim: int = 128) -> Workload:
    """8B-dLLM layer: batch 1, MHA H=32, d=128, prefix 4096, block 32, 32 steps, tau=4.

    Q ~ N(0,1).  Prefix and block K, V ~ s_h * N(0,1) with one s_h ~ U(0.5, 2) per
    head, shared by K and V.  Each step 1..S-1 redraws k = clamp(Poisson(2), 1, 4)
    distinct block tokens (the pages give "1-4 tokens, Poisson mean 2")."""
    rng = np.random.default_rng(seed)
    p = make_problem([np.arange(block)], [prefix], [block], heads, heads, head_dim)
    s_h = rng.uniform(0.5, 2.0, size=heads).astype(np.float32)
    sc = s_h[:, None]  # broadcast over [H, d]
    k_out = normal_bf16(rng, (prefix, heads, head_dim), sc)
    v_out = normal_bf16(rng, (prefix, heads, head_dim), sc)
    st = _BlockState(rng, p, 1.0, sc)
    out = [st.step_input([block])]
    for _ in range(1, steps):
        k = int(min(max(rng.poisson(2.0), 1), 4))
        _redraw_schedule(rng, p, st, [k])
        out.append(st.step_input([k]))
    return Workload("dllm_layer", p, k_out, v_out, out, tau=4, gamma=0.0, flags=GATE_TAU,
                    notes="H32 d128 prefix4096 block32; K,V scaled per head U(0.5,2); "
                          "k=clamp(Poisson(2),1,4) redraws/step; tau=4")


def long_context_gqa(seed: int = 1002, steps: int = 16, batch: int = 8, prefix: int = 32768,
                     block: int = 64, heads_q: int = 32, heads_kv: int = 8,
                     head_dim: int = 128, active: int = 32, force: int = FORCE_REUSE) -> Workload:
    """Long-context GQA: batch 8, H_q=32, H_kv=8, d=128, prefix 32768, block 64, 16 steps.

    A fixed seeded 32-of-64 set of query rows per sequence is active (the other
    rows are locked, SureLock style: no query, but their K/V stay in the block).
    Every step redraws Q/K/V of the active rows.  ``force`` picks the comparison
    arm: FORCE_RECOMPUTE (dense every step) or FORCE_REUSE (reuse after step 0)."""
    rng = np.random.default_rng(seed)
    rows = [np.sort(rng.permutation(block)[:active]) for _ in range(batch)]
    p = make_problem(rows, [prefix] * batch, [block] * batch, heads_q, heads_kv, head_dim)
    k_out = normal_bf16(rng, (p.total_kv_out, heads_kv, head_dim))
    v_out = normal_bf16(rng, (p.total_kv_out, heads_kv, head_dim))
    st = _BlockState(rng, p, 1.0, 1.0)
    act_tokens = np.concatenate([r + p.cu_seqlens_kv_in[b] for b, r in enumerate(rows)])
    out = [st.step_input([active] * batch)]
    for _ in range(1, steps):
        st.redraw(act_tokens)
        out.append(st.step_input([active] * batch))
    return Workload("long_context_gqa", p, k_out, v_out, out, tau=0, gamma=0.0, flags=force,
                    notes="b8 Hq32 Hkv8 d128 prefix32768 block64, 32/64 rows active; "
                          "active rows redrawn every step")


def varlen_branches(seed: int = 1003, steps: int = 8, blocks=(4, 8, 16, 32, 64, 128),
                    prefix: int = 2048, heads: int = 32, head_dim: int = 128) -> Workload:
    """One request, 6 branches (block sizes 4..128), each with its own 2048-token
    prefix, H=32, d=128, 8 steps.  All block rows are active and packed varlen.
    Per branch and step: M_b = clamp(Poisson(2), 1, B_b) redraws, tau=4."""
    rng = np.random.default_rng(seed)
    p = make_problem([np.arange(B) for B in blocks], [prefix] * len(blocks), list(blocks),
                     heads, heads, head_dim)
    k_out = normal_bf16(rng, (p.total_kv_out, heads, head_dim))
    v_out = normal_bf16(rng, (p.total_kv_out, heads, head_dim))
    st = _BlockState(rng, p, 1.0, 1.0)
    out = [st.step_input(list(blocks))]
    for _ in range(1, steps):
        ks = [int(min(max(rng.poisson(2.0), 1), B)) for B in blocks]
        _redraw_schedule(rng, p, st, ks)
        out.append(st.step_input(ks))
    return Workload("varlen_branches", p, k_out, v_out, out, tau=4, gamma=0.0, flags=GATE_TAU,
                    notes="6 branches B=4..128, prefix 2048 each, H32 d128; per-branch tau=4")


def video(seed: int = 1004, steps: int = 10, block: int = 1560, prefix_blocks: int = 6,
          heads: int = 40, head_dim: int = 128, gamma: float = 0.95,
          sigma_lo: float = 0.02, sigma_hi: float = 0.5) -> Workload:
    """Video-shaped: batch 1, H=40, d=128, block 1560 query tokens, prefix 6 blocks
    (9360 tokens), 10 steps, per-head cosine gate gamma=0.95, tau gate off.

    Prefix and initial block Q, K, V ~ N(0,1).  Each step perturbs the block Q/K/V
    of head h with step noise sigma_h in variance-preserving form,
    x <- (x + sigma_h * N(0,1)) / sqrt(1 + sigma_h^2) (float32 state, rounded to
    bf16 after each step), so the activations keep their N(0,1) scale from step to
    step (a denoising step does not inflate them) while consecutive steps of a head
    have cosine about 1 / sqrt(1 + sigma_h^2); a seeded random half of the heads
    gets sigma=0.02 (cosine 0.9998 per step), the other half sigma=0.5 (0.894)."""
    rng = np.random.default_rng(seed)
    N = prefix_blocks * block
    p = make_problem([np.arange(block)], [N], [block], heads, heads, head_dim)
    k_out = normal_bf16(rng, (N, heads, head_dim))
    v_out = normal_bf16(rng, (N, heads, head_dim))
    lo = np.zeros(heads, dtype=bool)
    lo[rng.permutation(heads)[: heads // 2]] = True
    sigma = np.where(lo, sigma_lo, sigma_hi).astype(np.float32)
    q = rng.standard_normal((block, heads, head_dim), dtype=np.float32)
    k = rng.standard_normal((block, heads, head_dim), dtype=np.float32)
    v = rng.standard_normal((block, heads, head_dim), dtype=np.float32)

    def snap():
        return StepInput(q=f32_to_bf16_bits(q), k_in=f32_to_bf16_bits(k), v_in=f32_to_bf16_bits(v),
                         n_updated=np.array([block], np.int32), problem=p)

    keep = (1.0 / np.sqrt(1.0 + sigma.astype(np.float64) ** 2)).astype(np.float32)
    out = [snap()]
    for _ in range(1, steps):
        for x in (q, k, v):
            x += sigma[None, :, None] * rng.standard_normal(x.shape, dtype=np.float32)
            x *= keep[None, :, None]
        out.append(snap())
    w = Workload("video", p, k_out, v_out, out, tau=0, gamma=gamma, flags=GATE_HEAD,
                 notes="H40 d128 block1560 prefix9360; variance-preserving step noise sigma 0.02/0.5 on halves; "
                       "gamma=0.95")
    w.sigma = sigma  # type: ignore[attr-defined]
    return w


def locking_tiny(seed: int = 1010, steps: int = 5, block: int = 48, prefix: int = 96,
                 heads_q: int = 4, heads_kv: int = 2, head_dim: int = 64, redraws=(3, 3)) -> Workload:
    """SureLock-style monotone locking on a small GQA problem (two sequences).

    Every step locks a few more rows (the active set only shrinks), redraws the
    Q/K/V of ``redraws[b]`` still-active rows of sequence b, and keeps tau gating
    on (tau = 4: with the default 3 redraws both sequences reuse after step 0; with
    (3, 5) the second sequence recomputes at every step and the first reuses)."""
    rng = np.random.default_rng(seed)
    active = [np.arange(block), np.arange(block - 8)]
    p0 = make_problem(active, [prefix, prefix + 37], [block, block - 8], heads_q, heads_kv, head_dim)
    k_out = normal_bf16(rng, (p0.total_kv_out, heads_kv, head_dim))
    v_out = normal_bf16(rng, (p0.total_kv_out, heads_kv, head_dim))
    st = _BlockState(rng, p0, 1.0, 1.0)
    out = [st.step_input([block, block - 8], p0)]
    for _ in range(1, steps):
        new_active = []
        for a in active:
            drop = rng.choice(len(a), size=min(5, len(a)), replace=False)
            new_active.append(np.sort(np.delete(a, drop)))
        active = new_active
        p = make_problem(active, [prefix, prefix + 37], [block, block - 8], heads_q, heads_kv, head_dim)
        toks = []
        for b, a in enumerate(active):
            sel = rng.choice(a, size=min(int(redraws[b]), len(a)), replace=False) + p.cu_seqlens_kv_in[b]
            toks.append(np.sort(sel))
        st.redraw(np.concatenate(toks))
        out.append(st.step_input([len(t) for t in toks], p))
    return Workload("locking_tiny", p0, k_out, v_out, out, tau=4, gamma=0.0, flags=GATE_TAU,
                    notes="2 seqs, GQA 4/2, d64, monotone locking, 3 redraws/step")


def next_block(w: Workload, seed: int, steps: int = 4, redraws: int = 2, name: str = "") -> Workload:
    """Inputs of the block that follows ``w``'s: same block lengths and the same
    active block positions as ``w``'s first step, each sequence's prefix longer by
    its finished block (J_out grows by B_b tokens), fresh Q/K/V for the new block,
    and ``redraws`` updated tokens per sequence and step (tau gate as in ``w``).

    Shapes and draws only: k_out / v_out are left as None -- the grown prefix (the
    old prefix followed by the finished block's K/V) is made by the block
    transition itself."""
    rng = np.random.default_rng(seed)
    p1 = w.steps[0].problem
    lens_out = p1.lens("out") + p1.lens("in")
    rows = [p1.q_rows[p1.cu_seqlens_q[b]:p1.cu_seqlens_q[b + 1]] for b in range(p1.num_seqs)]
    p = make_problem(rows, lens_out, p1.lens("in"), p1.num_heads_q, p1.num_heads_kv, p1.head_dim,
                     p1.softmax_scale)
    st = _BlockState(rng, p, 1.0, 1.0)
    out = [st.step_input(p.lens("in"))]
    for _ in range(1, steps):
        toks = []
        for b, r in enumerate(rows):
            k = min(redraws, len(r))
            if k:
                toks.append(np.sort(rng.choice(r, size=k, replace=False)) + p.cu_seqlens_kv_in[b])
        st.redraw(np.concatenate(toks) if toks else np.zeros(0, np.int64))
        out.append(st.step_input([min(redraws, len(r)) for r in rows]))
    return Workload(name or w.name + "_next_block", p, None, None, out, tau=w.tau, gamma=w.gamma, flags=w.flags,
                    notes="the block after " + w.name)


def first_sequences(w: Workload, n: int) -> Workload:
    """The same workload restricted to its first ``n`` sequences (input slicing only:
    the index arrays, Q rows, block and prefix K/V and update counts of those
    sequences).  Used to time the CPU oracle on a bounded sample of a batch whose
    sequences all have the same shape."""
    def cut(p: Problem) -> Problem:
        return Problem(num_seqs=n, num_heads_q=p.num_heads_q, num_heads_kv=p.num_heads_kv, head_dim=p.head_dim,
                       softmax_scale=p.softmax_scale, cu_seqlens_q=p.cu_seqlens_q[:n + 1].copy(),
                       q_rows=p.q_rows[:int(p.cu_seqlens_q[n])].copy(),
                       cu_seqlens_kv_out=p.cu_seqlens_kv_out[:n + 1].copy(),
                       cu_seqlens_kv_in=p.cu_seqlens_kv_in[:n + 1].copy())
    p0 = cut(w.problem)
    steps = []
    for st in w.steps:
        p = cut(st.problem)
        steps.append(StepInput(q=st.q[:p.total_q], k_in=st.k_in[:p.total_kv_in], v_in=st.v_in[:p.total_kv_in],
                               n_updated=st.n_updated[:n].copy(), problem=p))
    return dataclasses.replace(w, problem=p0, k_out=w.k_out[:p0.total_kv_out], v_out=w.v_out[:p0.total_kv_out],
                               steps=steps)


NAMED = {
    "tiny": tiny,
    "dllm_layer": dllm_layer,
    "long_context_gqa": long_context_gqa,
    "varlen_branches": varlen_branches,
    "video": video,
}
