"""Sparse-residual FlashBlock on the device (fb_sparse_layout + fb_step) against the
oracle's own partition and policy (needs a B200)."""
import dataclasses

import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, run_policy_gpu, torch_and_binding
from oracle import sparse

pytestmark = pytest.mark.gpu


def _selection(prefix_lens, seed=7):
    """Attention sink (first 64 keys), local window (last 256) and 32 seeded keys in
    between, per sequence."""
    rng = np.random.default_rng(seed)
    out = []
    for n in prefix_lens:
        mid = rng.choice(np.arange(64, n - 256), size=32, replace=False)
        out.append(np.unique(np.concatenate([np.arange(64), mid, np.arange(n - 256, n)])))
    return out


def _device_layout(B, torch, p, sel, k_out, v_out, k_in, v_in):
    cu_sel = np.concatenate([[0], np.cumsum([len(s) for s in sel])]).astype(np.int32)
    total_sel = int(cu_sel[-1])
    Hk, d = p.num_heads_kv, p.head_dim
    k_res = torch.empty((p.total_kv_out - total_sel, Hk, d), dtype=torch.bfloat16, device="cuda")
    v_res = torch.empty_like(k_res)
    k_ext = torch.empty((p.total_kv_in + total_sel, Hk, d), dtype=torch.bfloat16, device="cuda")
    v_ext = torch.empty_like(k_ext)
    cu_o = torch.full((p.num_seqs + 1,), -1, dtype=torch.int32, device="cuda")
    cu_i = torch.full((p.num_seqs + 1,), -1, dtype=torch.int32, device="cuda")
    B.sparse_layout(B.DeviceProblem(p), torch.as_tensor(cu_sel).cuda(),
                    torch.as_tensor(np.concatenate(sel).astype(np.int32)).cuda(), total_sel,
                    B.bf16_tensor(k_out), B.bf16_tensor(v_out), B.bf16_tensor(k_in), B.bf16_tensor(v_in),
                    k_res, v_res, k_ext, v_ext, cu_o, cu_i)
    torch.cuda.synchronize()
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return bits(k_res), bits(v_res), bits(k_ext), bits(v_ext), cu_o.cpu().numpy(), cu_i.cpu().numpy()


def test_sparse_residual_gqa():
    torch, B = torch_and_binding()
    w = W.long_context_gqa(steps=3, batch=2, prefix=1024 + 37)
    sel = _selection(np.diff(w.problem.cu_seqlens_kv_out))
    # the layout: bit-exact against the oracle's partition, for every step's block
    gpu_steps = []
    for st in w.steps:
        kr, vr, ke, ve, cu_o, cu_i = _device_layout(B, torch, st.problem, sel, w.k_out, w.v_out, st.k_in, st.v_in)
        p2, okr, ovr, oke, ove = sparse.rearrange(st.problem, w.k_out, w.v_out, st.k_in, st.v_in, sel)
        assert np.array_equal(kr, okr) and np.array_equal(vr, ovr)
        assert np.array_equal(ke, oke) and np.array_equal(ve, ove)
        assert np.array_equal(cu_o, p2.cu_seqlens_kv_out) and np.array_equal(cu_i, p2.cu_seqlens_kv_in)
        gpu_steps.append(dataclasses.replace(st, k_in=ke, v_in=ve,
                                             problem=dataclasses.replace(st.problem, cu_seqlens_kv_out=cu_o,
                                                                         cu_seqlens_kv_in=cu_i)))
    assert B.device_status() == 0
    # the step on the device-built layout against the oracle's sparse-residual policy
    gw = dataclasses.replace(w, problem=gpu_steps[0].problem, k_out=kr, v_out=vr, steps=gpu_steps)
    gpu, _ = run_policy_gpu(gw)
    ref = sparse.run_sparse_residual(w, sel, with_exact=True)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}: decisions differ"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"sparse residual step {s}")
    assert ref[0].reuse_error < 1e-12 and not ref[1].recompute.any()


def test_sparse_layout_rejects_a_bad_selection():
    """A selection that is not increasing is refused on the device (status), and the
    other sequence is still laid out."""
    torch, B = torch_and_binding()
    w = W.long_context_gqa(steps=1, batch=2, prefix=300, heads_q=8, heads_kv=2)
    st = w.steps[0]
    sel = [np.array([5, 3]), np.array([0, 299])]
    kr, vr, ke, ve, cu_o, cu_i = _device_layout(B, torch, st.problem, sel, w.k_out, w.v_out, st.k_in, st.v_in)
    assert B.device_status() == 1  # FB_ERR_INVALID_ARG recorded
    good = [np.array([], dtype=np.int64), np.array([0, 299])]
    _, okr, _, oke, _ = sparse.rearrange(st.problem, w.k_out, w.v_out, st.k_in, st.v_in, good)
    # the second sequence: residual rows 298.. on the device (the first sequence's
    # 300 - 2), 300.. in the oracle (no selection there); likewise 66.. and 64.. of J_in'
    assert np.array_equal(kr[298:], okr[300:]) and np.array_equal(ke[64 + 2:], oke[64:])
