"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and
compare it with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np

# Tolerances for bf16 inputs with fp32 accumulation.
A_MAX_ABS = 2e-2
A_MEAN_ABS = 1e-3
L_ABS = 1e-3


def torch_and_binding():
    import torch
    from cached_split_attention_b200 import binding as B
    return torch, B


def bf16_to_f64_torch(t):
    return t.float().double().cpu().numpy()


def assert_close(a_gpu, a_ref, l_gpu, l_ref, what="", a_max=A_MAX_ABS, a_mean=A_MEAN_ABS, l_abs=L_ABS):
    a_gpu = np.asarray(a_gpu, dtype=np.float64)
    a_ref = np.asarray(a_ref, dtype=np.float64)
    sel = ~np.isnan(a_ref)
    assert sel.any(), f"{what}: nothing to compare"
    assert np.all(np.isfinite(a_gpu[sel])), f"{what}: non-finite A from the GPU"
    err = np.abs(a_gpu[sel] - a_ref[sel])
    assert err.max() <= a_max, f"{what}: A max-abs {err.max():.3e} > {a_max}"
    assert err.mean() <= a_mean, f"{what}: A mean-abs {err.mean():.3e} > {a_mean}"
    if l_ref is not None:
        l_gpu = np.asarray(l_gpu, dtype=np.float64)
        l_ref = np.asarray(l_ref, dtype=np.float64)
        ls = ~np.isnan(l_ref)
        both_inf = np.isneginf(l_ref[ls]) & np.isneginf(l_gpu[ls])
        with np.errstate(invalid="ignore"):
            le = np.where(both_inf, 0.0, np.abs(l_gpu[ls] - l_ref[ls]))
        assert np.all(np.isfinite(le)), f"{what}: L mismatch in infinities"
        assert le.max(initial=0) <= l_abs, f"{what}: L max-abs {le.max():.3e} > {l_abs}"
    return float(err.max()), float(err.mean())


def workspace_for(steps_problems, out_splits=0, device="cuda"):
    torch, B = torch_and_binding()
    size = 16
    for p in steps_problems:
        size = max(size, B.workspace_size(B.DeviceProblem(p, device, out_splits)))
    ws = torch.empty(size, dtype=torch.uint8, device=device)
    B.workspace_init(ws)
    return ws


def run_policy_gpu(w, flags=None, out_splits=0, head_reuse_in=None, device="cuda", keep=True, cache=None,
                   k_out=None, v_out=None, kv_out_skip=None):
    """Run a workload's steps through fb_step (on ``cache`` when given, else on a new
    empty one; on the device prefix ``k_out``/``v_out`` when given, else on w's
    uploaded); returns per-step dicts of numpy arrays and the cache."""
    torch, B = torch_and_binding()
    flags = w.flags if flags is None else flags
    p0 = w.problem
    cache = cache if cache is not None else B.Cache(p0, device, with_q_ref=True)
    k_out = B.bf16_tensor(w.k_out, device) if k_out is None else k_out
    v_out = B.bf16_tensor(w.v_out, device) if v_out is None else v_out
    ws = workspace_for([st.problem for st in w.steps], out_splits, device)
    prm = B.params(w.tau, w.gamma, flags)
    out = []
    for s, st in enumerate(w.steps):
        p = st.problem
        dp = B.DeviceProblem(p, device, out_splits, kv_out_skip=kv_out_skip)
        q = B.bf16_tensor(st.q, device)
        k_in = B.bf16_tensor(st.k_in, device)
        v_in = B.bf16_tensor(st.v_in, device)
        n_upd = torch.as_tensor(st.n_updated, dtype=torch.int32).to(device)
        a_full = torch.full((max(p.total_q, 1), p.num_heads_q, p.head_dim), float("nan"),
                            dtype=torch.bfloat16, device=device)
        l_full = torch.full((max(p.total_q, 1), p.num_heads_q), float("nan"), dtype=torch.float32, device=device)
        dec = torch.full((p.num_seqs, p.num_heads_q), 7, dtype=torch.uint8, device=device)
        hr = None
        if head_reuse_in is not None and head_reuse_in[s] is not None:
            hr = torch.as_tensor(head_reuse_in[s].astype(np.uint8)).to(device)
        B.step(dp, prm, cache, q, k_in, v_in, k_out, v_out, n_upd, a_full, ws, l_full=l_full,
               head_reuse_in=hr, decision_out=dec)
        torch.cuda.synchronize()
        if keep:
            out.append(dict(a_full=bf16_to_f64_torch(a_full[:p.total_q]),
                            l_full=l_full[:p.total_q].double().cpu().numpy(),
                            decision=dec.cpu().numpy().astype(bool)))
    status = B.device_status()
    assert status == 0, f"device status {status}"
    return out, cache
