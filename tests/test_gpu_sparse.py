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
    """fb_sparse_layout on the device: J_in' rows, the prefix skip mask, the J_in' offsets."""
    cu_sel = np.concatenate([[0], np.cumsum([len(s) for s in sel])]).astype(np.int32)
    total_sel = int(cu_sel[-1])
    Hk, d = p.num_heads_kv, p.head_dim
    k_ext = torch.empty((p.total_kv_in + total_sel, Hk, d), dtype=torch.bfloat16, device="cuda")
    v_ext = torch.empty_like(k_ext)
    skip = torch.full(((p.total_kv_out + 31) // 32,), -1, dtype=torch.int32, device="cuda")
    cu_i = torch.full((p.num_seqs + 1,), -1, dtype=torch.int32, device="cuda")
    B.sparse_layout(B.DeviceProblem(p), torch.as_tensor(cu_sel).cuda(),
                    torch.as_tensor(np.concatenate(sel).astype(np.int32)).cuda(), total_sel,
                    B.bf16_tensor(k_out), B.bf16_tensor(v_out), B.bf16_tensor(k_in), B.bf16_tensor(v_in),
                    k_ext, v_ext, skip, cu_i)
    torch.cuda.synchronize()
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return bits(k_ext), bits(v_ext), skip, cu_i.cpu().numpy()


def _selected_tokens(p, sel):
    """Global prefix rows of the selected keys."""
    return np.concatenate([int(p.cu_seqlens_kv_out[b]) + np.asarray(s, dtype=np.int64) for b, s in enumerate(sel)])


def test_sparse_residual_gqa():
    torch, B = torch_and_binding()
    w = W.long_context_gqa(steps=3, batch=2, prefix=1024 + 37)
    sel = _selection(np.diff(w.problem.cu_seqlens_kv_out))
    # the layout: J_in' bit-exact against the oracle's partition for every step's
    # block, and the skip mask marks exactly the selected prefix rows
    layouts = []
    for st in w.steps:
        ke, ve, skip, cu_i = _device_layout(B, torch, st.problem, sel, w.k_out, w.v_out, st.k_in, st.v_in)
        p2, _, _, oke, ove = sparse.rearrange(st.problem, w.k_out, w.v_out, st.k_in, st.v_in, sel)
        assert np.array_equal(ke, oke) and np.array_equal(ve, ove)
        assert np.array_equal(cu_i, p2.cu_seqlens_kv_in)
        words = skip.cpu().numpy().view(np.uint32)
        bits = np.unpackbits(words.view(np.uint8), bitorder="little")[:st.problem.total_kv_out]
        want = np.zeros(st.problem.total_kv_out, dtype=np.uint8)
        want[_selected_tokens(st.problem, sel)] = 1
        assert np.array_equal(bits, want)
        layouts.append((ke, ve, skip, cu_i))
    assert B.device_status() == 0
    # fb_step on (prefix with the skip mask, J_in') against the oracle's sparse-residual
    # policy, which attends to the materialised residual prefix
    gpu = []
    cache = B.Cache(dataclasses.replace(w.problem, cu_seqlens_kv_in=layouts[0][3]), "cuda", with_q_ref=True)
    k_out, v_out = B.bf16_tensor(w.k_out), B.bf16_tensor(w.v_out)
    for st, (ke, ve, skip, cu_i) in zip(w.steps, layouts):
        p2 = dataclasses.replace(st.problem, cu_seqlens_kv_in=cu_i)
        gw = dataclasses.replace(w, problem=p2, steps=[dataclasses.replace(st, k_in=ke, v_in=ve, problem=p2)])
        out, cache = run_policy_gpu(gw, cache=cache, k_out=k_out, v_out=v_out, kv_out_skip=skip)
        gpu += out
    ref = sparse.run_sparse_residual(w, sel, with_exact=True)
    for s, (g, r) in enumerate(zip(gpu, ref)):
        assert np.array_equal(g["decision"], r.recompute), f"step {s}: decisions differ"
        assert_close(g["a_full"], r.a_full, g["l_full"], r.l_full, f"sparse residual step {s}")
    assert ref[0].reuse_error < 1e-12 and not ref[1].recompute.any()


def test_sparse_skip_mask_in_every_prefix_kernel():
    """The skip mask in the prefix pass of each kernel family (warp MMA: the dLLM
    shape; tcgen05 one tile: GQA groups of 128 rows; tcgen05 two tiles: a 300-token
    MHA block), forced recompute with a fresh cache, against full attention over the
    oracle's partition."""
    torch, B = torch_and_binding()
    cases = [W.dllm_layer(steps=1, prefix=700), W.long_context_gqa(steps=1, batch=2, prefix=333),
             W.video(steps=1, block=300, prefix_blocks=1, heads=4)]
    for w in cases:
        rng = np.random.default_rng(3)
        p, st = w.problem, w.steps[0]
        sel = [np.unique(rng.choice(int(n), size=min(int(n), 90), replace=False)) for n in p.lens("out")]
        ke, ve, skip, cu_i = _device_layout(B, torch, p, sel, w.k_out, w.v_out, st.k_in, st.v_in)
        p2 = dataclasses.replace(p, cu_seqlens_kv_in=cu_i)
        gw = dataclasses.replace(w, problem=p2, steps=[dataclasses.replace(st, k_in=ke, v_in=ve, problem=p2)])
        gpu, _ = run_policy_gpu(gw, flags=W.FORCE_RECOMPUTE, kv_out_skip=skip)
        ref = sparse.run_sparse_residual(w, sel, flags=W.FORCE_RECOMPUTE, with_exact=True)
        assert ref[0].reuse_error < 1e-12
        assert_close(gpu[0]["a_full"], ref[0].a_full, gpu[0]["l_full"], ref[0].l_full, f"{w.name} skip mask")


def test_sparse_layout_rejects_a_bad_selection():
    """A selection that is not increasing is refused on the device (status), and the
    other sequence is still laid out."""
    torch, B = torch_and_binding()
    w = W.long_context_gqa(steps=1, batch=2, prefix=300, heads_q=8, heads_kv=2)
    st = w.steps[0]
    sel = [np.array([5, 3]), np.array([0, 299])]
    ke, ve, skip, cu_i = _device_layout(B, torch, st.problem, sel, w.k_out, w.v_out, st.k_in, st.v_in)
    assert B.device_status() == 1  # FB_ERR_INVALID_ARG recorded
    good = [np.array([], dtype=np.int64), np.array([0, 299])]
    _, _, _, oke, _ = sparse.rearrange(st.problem, w.k_out, w.v_out, st.k_in, st.v_in, good)
    # the second sequence's J_in' starts at 64 + 2 on the device (the first sequence's
    # two selected rows are counted in cu_sel), at 64 in the oracle (no selection there)
    assert np.array_equal(ke[64 + 2:], oke[64:])
    words = skip.cpu().numpy().view(np.uint32)
    bits = np.unpackbits(words.view(np.uint8), bitorder="little")[:st.problem.total_kv_out]
    assert bits.sum() == 2 and bits[300] == 1 and bits[599] == 1
