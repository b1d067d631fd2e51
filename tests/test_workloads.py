"""The seeded input generators: determinism, shapes and schedule recipes (CPU)."""
import numpy as np

from cached_split_attention_b200 import workloads as W


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-9, -2.5, 1.00390625], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert back.tolist() == [1.0, 1.0, 1.0 + 2**-7, -2.5, 1.0]


def test_deterministic():
    a, b = W.tiny(), W.tiny()
    assert np.array_equal(a.k_out, b.k_out)
    for x, y in zip(a.steps, b.steps):
        assert np.array_equal(x.q, y.q) and np.array_equal(x.v_in, y.v_in)
    c = W.tiny(seed=7)
    assert not np.array_equal(a.k_out, c.k_out)


def test_tiny_recipe():
    w = W.tiny()
    p = w.problem
    assert (p.num_heads_q, p.head_dim, p.total_kv_out, p.total_kv_in, p.total_q) == (4, 64, 256, 32, 32)
    assert len(w.steps) == 4 and w.tau == 8
    for s in range(1, 4):
        changed = np.any(w.steps[s].k_in != w.steps[s - 1].k_in, axis=(1, 2))
        assert changed.sum() <= 4 and w.steps[s].n_updated[0] == 4


def test_dllm_schedule_counts():
    w = W.dllm_layer(prefix=64)
    ks = [int(s.n_updated[0]) for s in w.steps[1:]]
    assert len(w.steps) == 32 and all(1 <= k <= 4 for k in ks)
    assert 4 in ks and 1 in ks
    for s in range(1, 32):
        changed = np.any(w.steps[s].q != w.steps[s - 1].q, axis=(1, 2)).sum()
        assert changed <= ks[s - 1]


def test_gqa_active_rows():
    w = W.long_context_gqa(prefix=128, steps=2)
    p = w.problem
    assert p.num_seqs == 8 and p.num_heads_q == 32 and p.num_heads_kv == 8
    assert np.all(np.diff(p.cu_seqlens_q) == 32)
    for b in range(8):
        rows = p.q_rows[p.cu_seqlens_q[b]:p.cu_seqlens_q[b + 1]]
        assert len(set(rows.tolist())) == 32 and rows.min() >= 0 and rows.max() < 64


def test_varlen_offsets():
    w = W.varlen_branches(prefix=16, steps=2)
    p = w.problem
    assert p.cu_seqlens_q.tolist() == [0, 4, 12, 28, 60, 124, 252]
    assert p.cu_seqlens_kv_out.tolist() == [16 * i for i in range(7)]


def test_video_sigma_halves():
    w = W.video(steps=2, block=16, prefix_blocks=2, heads=8)
    assert (w.sigma < 0.1).sum() == 4 and w.flags == W.GATE_HEAD


def test_video_step_noise_keeps_the_scale():
    """The step noise is variance-preserving: after 9 steps the block Q/K/V of every
    head still have unit variance (a cumulative walk would reach 1 + 9 sigma^2 =
    3.25 for sigma = 0.5), and a sigma = 0.5 head's queries at consecutive steps
    have cosine close to 1 / sqrt(1 + 0.25) = 0.894."""
    from oracle.attention import bf16_to_f64
    w = W.video(steps=10, block=256, prefix_blocks=1, heads=8)
    q0, q9 = bf16_to_f64(w.steps[0].q), bf16_to_f64(w.steps[9].q)
    for x in (q9, bf16_to_f64(w.steps[9].k_in), bf16_to_f64(w.steps[9].v_in)):
        var = x.var(axis=(0, 2))
        assert np.all(np.abs(var - 1.0) < 0.05), var
    hi = np.flatnonzero(w.sigma > 0.1)[0]
    a, b = bf16_to_f64(w.steps[1].q)[:, hi].ravel(), q0[:, hi].ravel()
    cos = a @ b / np.sqrt((a @ a) * (b @ b))
    assert abs(cos - 1 / np.sqrt(1.25)) < 0.01, cos


def test_dllm_default_recompute_steps():
    """The 8B-dLLM layer as the bench runs it (seed 1001): with tau = 4 the steps
    that recompute are 0, 2, 7, 12 and 25 (k = clamp(Poisson(2), 1, 4) reaches 4
    at steps 2, 7, 12, 25)."""
    w = W.dllm_layer()
    ks = [int(s.n_updated[0]) for s in w.steps]
    assert [0] + [s for s in range(1, 32) if ks[s] >= w.tau] == [0, 2, 7, 12, 25]
