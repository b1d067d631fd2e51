"""Guard bands around every buffer the library writes (needs a B200).

Each output, cache and workspace tensor is carved out of a larger byte buffer,
between two 4 KiB bands of a canary byte.  After several steps through every
attention kernel (warp MMA; tensor cores with one and with two softmax threads
per row; the two-tile kernel with its similarity and work-order passes), on
recompute, reuse and lean-path steps with ragged shapes, every band must be
intact, the inputs unchanged and the device status clean, and the results must
still match the oracle: a write past either end of any buffer, or into an
input, fails here even where it would not change a compared value."""
import ctypes

import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, torch_and_binding
from oracle import attention, policy

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


class Guarded:
    """Tensors, each in its own byte buffer between two canary bands."""

    def __init__(self):
        self.bufs = []

    def tensor(self, shape, dtype, fill):
        torch, _ = torch_and_binding()
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        t = raw[GUARD:GUARD + n].view(dtype).view(shape)
        t.fill_(fill)
        self.bufs.append((raw, n))
        return t

    def damaged(self):
        """Indices of the buffers whose bands were written."""
        bad = []
        for i, (raw, n) in enumerate(self.bufs):
            if not (bool((raw[:GUARD] == CANARY).all()) and bool((raw[GUARD + n:] == CANARY).all())):
                bad.append(i)
        return bad


class GuardedCache:
    """The caller's FlashBlock cache, every array guarded."""

    def __init__(self, g, problem):
        torch, B = torch_and_binding()
        T, H, d = max(problem.total_kv_in, 1), problem.num_heads_q, problem.head_dim
        S = max(problem.num_seqs, 1)
        self.a_out = g.tensor((T, H, d), torch.float32, 0.0)
        self.l_out = g.tensor((T, H), torch.float32, 0.0)
        self.valid = g.tensor((S, H), torch.uint8, 0)
        self.q_ref = g.tensor((T, H, d), torch.bfloat16, 0.0)
        self.m_acc = g.tensor((S, H), torch.int32, 0)
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        self.struct = B.FbCache(p(self.a_out), p(self.l_out), p(self.valid), p(self.q_ref), p(self.m_acc))

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def _guarded_episode(w, flags):
    torch, B = torch_and_binding()
    g = Guarded()
    p0 = w.problem
    cache = GuardedCache(g, p0)
    k_out = B.bf16_tensor(w.k_out)
    v_out = B.bf16_tensor(w.v_out)
    k_out0, v_out0 = k_out.clone(), v_out.clone()
    size = max(16, max(B.workspace_size(B.DeviceProblem(st.problem)) for st in w.steps))
    ws = g.tensor((size,), torch.uint8, 0)
    B.workspace_init(ws)
    prm = B.params(w.tau, w.gamma, flags)
    out = []
    for st in w.steps:
        p = st.problem
        dp = B.DeviceProblem(p)
        q, k_in, v_in = B.bf16_tensor(st.q), B.bf16_tensor(st.k_in), B.bf16_tensor(st.v_in)
        q0, k_in0, v_in0 = q.clone(), k_in.clone(), v_in.clone()
        cu = [dp.cu_q.clone(), dp.cu_out.clone(), dp.cu_in.clone()]
        n_upd = torch.as_tensor(st.n_updated, dtype=torch.int32).cuda()
        n_upd0 = n_upd.clone()
        rows = max(p.total_q, 1)
        a_full = g.tensor((rows, p.num_heads_q, p.head_dim), torch.bfloat16, float("nan"))
        l_full = g.tensor((rows, p.num_heads_q), torch.float32, float("nan"))
        dec = g.tensor((max(p.num_seqs, 1), p.num_heads_q), torch.uint8, 7)
        B.step(dp, prm, cache, q, k_in, v_in, k_out, v_out, n_upd, a_full, ws, l_full=l_full, decision_out=dec)
        torch.cuda.synchronize()
        for a, b in zip([q, k_in, v_in, n_upd, dp.cu_q, dp.cu_out, dp.cu_in], [q0, k_in0, v_in0, n_upd0, *cu]):
            assert torch.equal(a, b), f"{w.name}: an input was written"
        out.append(dict(a_full=a_full[:p.total_q].float().double().cpu().numpy(),
                        l_full=l_full[:p.total_q].double().cpu().numpy(),
                        decision=dec[:p.num_seqs].cpu().numpy().astype(bool)))
    assert torch.equal(k_out, k_out0) and torch.equal(v_out, v_out0), f"{w.name}: the prefix was written"
    assert B.device_status() == 0
    assert not g.damaged(), f"{w.name}: guard bands written around buffers {g.damaged()}"
    return out


# (id, workload, flags (None: the workload's gates), kernel the plan picks, threads per CTA)
CASES = [
    ("warp_mma_d64", lambda: W.tiny(), None, "attn_kernel", 256),
    ("warp_mma_dllm", lambda: W.dllm_layer(steps=4, prefix=1000), None, "attn_kernel", 256),
    ("tensor_core_gqa_reuse", lambda: W.long_context_gqa(steps=3, batch=3, prefix=300), W.FORCE_REUSE,
     "tc_attn_kernel", 192),
    ("tensor_core_gqa_recompute", lambda: W.long_context_gqa(steps=2, batch=3, prefix=300), W.FORCE_RECOMPUTE,
     "tc_attn_kernel", 192),
    ("tensor_core_two_threads_varlen", lambda: W.varlen_branches(steps=4, prefix=337), None, "tc_attn_kernel", 320),
    ("two_tile_video", lambda: W.video(steps=3, block=300, prefix_blocks=1, heads=4), None, "tc2_attn_kernel", 320),
]


@pytest.mark.parametrize("name,make,flags,kernel,threads", CASES, ids=[c[0] for c in CASES])
def test_fused_step_writes_only_its_buffers(name, make, flags, kernel, threads):
    _, B = torch_and_binding()
    w = make()
    plan = B.plan_query(B.DeviceProblem(w.problem))
    assert (plan["kernel_name"], plan["threads"]) == (kernel, threads)
    flags = w.flags if flags is None else flags
    gpu = _guarded_episode(w, flags)
    ref = policy.run_policy(w, flags=flags)
    for s, (a, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(a["decision"], r.recompute), f"{name} step {s}: decisions differ"
        assert_close(a["a_full"], r.a_full, a["l_full"], r.l_full, f"{name} step {s}")


def test_unfused_passes_write_only_their_buffers():
    """fb_out_attn (every other head masked; it writes by cache row), fb_in_attn and
    fb_merge on a ragged GQA problem with locked rows, each output and the workspace
    guarded; cache rows of locked tokens and masked heads stay untouched."""
    torch, B = torch_and_binding()
    w = W.long_context_gqa(steps=1, batch=3, prefix=300)
    st = w.steps[0]
    p = st.problem
    dp = B.DeviceProblem(p)
    g = Guarded()
    H, d, n, T = p.num_heads_q, p.head_dim, p.total_q, p.total_kv_in
    crow = policy.cache_rows(p)
    a_o = g.tensor((T, H, d), torch.float32, float("nan"))
    l_o = g.tensor((T, H), torch.float32, float("nan"))
    a_i = g.tensor((n, H, d), torch.float32, float("nan"))
    l_i = g.tensor((n, H), torch.float32, float("nan"))
    ws = g.tensor((max(16, B.workspace_size(dp)),), torch.uint8, 0)
    B.workspace_init(ws)
    mask = np.zeros((p.num_seqs, H), dtype=np.uint8)
    mask[:, ::2] = 1
    q = B.bf16_tensor(st.q)
    B.out_attn(dp, q, B.bf16_tensor(w.k_out), B.bf16_tensor(w.v_out), a_o, l_o, ws,
               head_mask=torch.as_tensor(mask).cuda())
    B.in_attn(dp, q, B.bf16_tensor(st.k_in), B.bf16_tensor(st.v_in), a_i, l_i)
    # merge the computed heads of the active rows
    rows = torch.as_tensor(crow).cuda()
    a_om, l_om = a_o[rows][:, ::2].contiguous(), l_o[rows][:, ::2].contiguous()
    a_im, l_im = a_i[:, ::2].contiguous(), l_i[:, ::2].contiguous()
    af = g.tensor(tuple(a_om.shape), torch.float32, float("nan"))
    ab = g.tensor(tuple(a_om.shape), torch.bfloat16, float("nan"))
    lf = g.tensor(tuple(l_om.shape), torch.float32, float("nan"))
    B.merge(a_om, l_om, a_im, l_im, a_full_f32=af, a_full_bf16=ab, l_full=lf)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert not g.damaged(), f"guard bands written around buffers {g.damaged()}"
    ao_h, lo_h = a_o.double().cpu().numpy(), l_o.double().cpu().numpy()
    written = np.zeros((T, H), dtype=bool)
    written[np.ix_(crow, np.arange(0, H, 2))] = True
    assert np.isnan(ao_h[~written]).all() and np.isnan(lo_h[~written]).all()
    ar, lr = attention.attend_problem(p, st.q, w.k_out, w.v_out, "out")
    ai, li = attention.attend_problem(p, st.q, st.k_in, st.v_in, "in")
    assert_close(ao_h[crow][:, ::2], ar[:, ::2], lo_h[crow][:, ::2], lr[:, ::2], "out pass")
    assert_close(a_i.double().cpu().numpy(), ai, l_i.double().cpu().numpy(), li, "in pass")
    fr, flr = attention.merge(ar, lr, ai, li)
    assert_close(af.double().cpu().numpy(), fr[:, ::2], lf.double().cpu().numpy(), flr[:, ::2], "merged")
