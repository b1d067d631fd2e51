"""CUDA path vs the fp64 oracle, kernel by kernel, through the C ABI (needs a B200)."""
import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, bf16_to_f64_torch, torch_and_binding
from oracle import attention, policy

pytestmark = pytest.mark.gpu


def _problems():
    """Small problems that still span several key tiles and end in ragged tails."""
    rng = np.random.default_rng(5)
    out = []
    # tiny: H4 d64, prefix 256, block 32
    out.append(("tiny", W.tiny().problem, 1.0))
    out.append(("tiny_sharp", W.tiny().problem, 32.0))
    # GQA g=2, ragged prefixes (not multiples of 64), shrunken active sets, q_rows permuted
    p = W.make_problem([[5, 0, 17, 3, 40], [1, 2]], [200, 37], [48, 40], 4, 2, 64)
    out.append(("gqa2_ragged_d64", p, 1.0))
    # d=128, GQA g=4, 3 sequences, one with no prefix, one with a single block key
    p = W.make_problem([np.arange(20), [0], rng.permutation(64)[:33]], [130, 0, 513], [20, 1, 64], 8, 2, 128)
    out.append(("gqa4_edge_d128", p, 1.0))
    # g=8 so rows of one token span a whole 16-row slab; a sequence with no active rows
    p = W.make_problem([np.arange(9), [], [3, 1]], [70, 64, 1], [9, 4, 5], 8, 1, 128)
    out.append(("gqa8_empty_rows", p, 2.0))
    # MHA with row tiles of 128 rows (several tiles per group)
    p = W.make_problem([np.arange(150)], [300], [150], 2, 2, 128)
    out.append(("mha_multi_tile", p, 1.0))
    # tensor-core path: 3 row tiles (128, 128, 44), 8 prefix chunks of 128 keys
    # (the last one 104 keys), 3 block chunks (the last one 44 keys)
    p = W.make_problem([np.arange(300)], [1000], [300], 2, 2, 128)
    out.append(("mha_tc_ragged", p, 1.0))
    # the same with sharp scores: the running max jumps, O is rescaled in TMEM
    out.append(("mha_tc_sharp", p, 40.0))
    # tensor-core path, GQA g=4: 2 sequences, 64 and 37 active rows in permuted
    # block order (256 and 148 rows), prefixes 777 and 129
    p = W.make_problem([rng.permutation(64), rng.permutation(80)[:37]], [777, 129], [64, 80], 8, 2, 128)
    out.append(("gqa4_tc_two_tiles", p, 1.0))
    return out


def _inputs(p, sharp, seed=11):
    rng = np.random.default_rng(seed)
    H, Hk, d = p.num_heads_q, p.num_heads_kv, p.head_dim
    s = sharp / np.sqrt(d) if sharp != 1.0 else 1.0
    q = W.normal_bf16(rng, (max(p.total_q, 0), H, d), s)
    ko = W.normal_bf16(rng, (p.total_kv_out, Hk, d), s)
    vo = W.normal_bf16(rng, (p.total_kv_out, Hk, d))
    ki = W.normal_bf16(rng, (p.total_kv_in, Hk, d), s)
    vi = W.normal_bf16(rng, (p.total_kv_in, Hk, d))
    return q, ko, vo, ki, vi


PROBLEMS = _problems()


@pytest.mark.parametrize("name,p,sharp", PROBLEMS, ids=[x[0] for x in PROBLEMS])
def test_in_attn(name, p, sharp):
    torch, B = torch_and_binding()
    q, ko, vo, ki, vi = _inputs(p, sharp)
    dp = B.DeviceProblem(p)
    a = torch.full((max(p.total_q, 1), p.num_heads_q, p.head_dim), float("nan"), device="cuda")
    l = torch.full((max(p.total_q, 1), p.num_heads_q), float("nan"), device="cuda")
    B.in_attn(dp, B.bf16_tensor(q), B.bf16_tensor(ki), B.bf16_tensor(vi), a, l)
    torch.cuda.synchronize()
    ar, lr = attention.attend_problem(p, q, ki, vi, "in")
    if p.total_q:
        assert_close(a[:p.total_q].double().cpu().numpy(), ar, l[:p.total_q].double().cpu().numpy(), lr, name)
    assert B.device_status() == 0


@pytest.mark.parametrize("splits", [1, 3, 0])
@pytest.mark.parametrize("name,p,sharp", PROBLEMS, ids=[x[0] for x in PROBLEMS])
def test_out_attn(name, p, sharp, splits):
    torch, B = torch_and_binding()
    q, ko, vo, ki, vi = _inputs(p, sharp)
    dp = B.DeviceProblem(p, out_splits=splits)
    ws = torch.empty(B.workspace_size(dp), dtype=torch.uint8, device="cuda")
    B.workspace_init(ws)
    T, H, d = p.total_kv_in, p.num_heads_q, p.head_dim
    a = torch.full((T, H, d), float("nan"), device="cuda")
    l = torch.full((T, H), float("nan"), device="cuda")
    # every other head of every sequence: masked heads must stay untouched
    mask = np.zeros((p.num_seqs, H), dtype=np.uint8)
    mask[:, ::2] = 1
    B.out_attn(dp, B.bf16_tensor(q), B.bf16_tensor(ko), B.bf16_tensor(vo), a, l, ws,
               head_mask=torch.as_tensor(mask).cuda())
    torch.cuda.synchronize()
    ar, lr = attention.attend_problem(p, q, ko, vo, "out")
    crow = policy.cache_rows(p)
    a_h = a.double().cpu().numpy()
    l_h = l.double().cpu().numpy()
    if p.total_q:
        on = np.zeros((p.total_q, H), dtype=bool)
        for b in range(p.num_seqs):
            on[p.cu_seqlens_q[b]:p.cu_seqlens_q[b + 1]] = mask[b][None, :] == 1
        ref_a = np.where(on[..., None], ar, np.nan)
        ref_l = np.where(on, lr, np.nan)
        assert_close(a_h[crow], ref_a, l_h[crow], ref_l, f"{name}/splits={splits}")
        # masked heads and inactive positions: still the NaN sentinel
        written = np.zeros((T, H), dtype=bool)
        rr, hh = np.nonzero(on)
        written[crow[rr], hh] = True
        assert np.all(np.isnan(l_h[~written])), "a masked head or an inactive position was written"
        assert np.all(np.isnan(a_h[~written])), "a masked head or an inactive position was written"
    assert B.device_status() == 0


def test_merge_kernel():
    torch, B = torch_and_binding()
    rng = np.random.default_rng(3)
    n, d = 1000, 96
    ao = rng.standard_normal((n, d)); ai = rng.standard_normal((n, d))
    lo = rng.standard_normal(n) * 5; li = rng.standard_normal(n) * 5
    lo[:10] = -np.inf
    li[5:15] = -np.inf
    lo[20] = 80.0; li[20] = -80.0
    t = lambda x: torch.as_tensor(x, dtype=torch.float32).cuda().contiguous()
    af = torch.empty((n, d), device="cuda")
    ab = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    lf = torch.empty(n, device="cuda")
    B.merge(t(ao), t(lo), t(ai), t(li), a_full_f32=af, a_full_bf16=ab, l_full=lf)
    torch.cuda.synchronize()
    ref_a, ref_l = attention.merge(np.float32(ao), np.float32(lo), np.float32(ai), np.float32(li))
    assert_close(af.double().cpu().numpy(), ref_a, lf.double().cpu().numpy(), ref_l, "merge f32", a_max=1e-5,
                 a_mean=1e-6, l_abs=1e-5)
    # the bf16 output is the fp32 result rounded to nearest even, bit for bit
    assert torch.equal(ab, af.to(torch.bfloat16))


def test_head_similarity():
    torch, B = torch_and_binding()
    w = W.video(steps=2, block=200, prefix_blocks=1, heads=6)
    p = w.problem
    dp = B.DeviceProblem(p)
    q_ref = B.bf16_tensor(w.steps[0].q)         # block positions == packed rows here
    q = B.bf16_tensor(w.steps[1].q)
    cos = torch.empty(p.num_seqs * p.num_heads_q, device="cuda")
    B.head_similarity(dp, q, q_ref, cos)
    torch.cuda.synchronize()
    ref = policy.head_cosine(p, attention.bf16_to_f64(w.steps[1].q), attention.bf16_to_f64(w.steps[0].q))
    assert np.abs(cos.double().cpu().numpy().reshape(ref.shape) - ref).max() < 1e-5
