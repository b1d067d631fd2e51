"""ctypes binding of libflashblock.so (include/flashblock.h).

Argument marshalling only: every step of the attention path runs in the CUDA
library.  Device memory and streams come from PyTorch.  Importing this module
fails loudly when the library is missing or does not export the ABI; there is no
fallback implementation.

Names mirror the C ABI without the ``fb_`` prefix (``step`` is ``fb_step``).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflashblock.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
GATE_TAU, GATE_HEAD, FORCE_RECOMPUTE, FORCE_REUSE, GATE_TAU_CUM = 1, 2, 4, 8, 16
CALL_STEP, CALL_OUT, CALL_IN = 0, 1, 2
KERNEL_NAMES = {0: "attn_kernel", 1: "tc_attn_kernel", 2: "tc2_attn_kernel"}


class FlashBlockError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"flashblock status {status}: {message}")
        self.status = status


class FbProblem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("num_heads_q", ctypes.c_int32),
        ("num_heads_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("cu_seqlens_q", ctypes.c_void_p), ("q_rows", ctypes.c_void_p),
        ("cu_seqlens_kv_out", ctypes.c_void_p), ("cu_seqlens_kv_in", ctypes.c_void_p),
        ("total_q", ctypes.c_int32), ("total_kv_out", ctypes.c_int32), ("total_kv_in", ctypes.c_int32),
        ("max_q", ctypes.c_int32), ("max_kv_out", ctypes.c_int32), ("max_kv_in", ctypes.c_int32),
        ("out_splits", ctypes.c_int32),
        ("kv_out_skip", ctypes.c_void_p),
    ]


class FbCache(ctypes.Structure):
    _fields_ = [("a_out", ctypes.c_void_p), ("l_out", ctypes.c_void_p),
                ("valid", ctypes.c_void_p), ("q_ref", ctypes.c_void_p), ("m_acc", ctypes.c_void_p)]


class FbParams(ctypes.Structure):
    _fields_ = [("tau", ctypes.c_int32), ("gamma", ctypes.c_float), ("flags", ctypes.c_uint32)]


class FbPlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("kernel", "rows_per_tile", "tiles", "work_items", "splits", "ctas",
                                              "threads", "smem_bytes", "keys_per_chunk", "num_sms",
                                              "lean_reuse", "lean_smem_bytes", "lean_early")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cached_split_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, vp, st = ctypes.POINTER(FbProblem), ctypes.c_void_p, ctypes.c_int
    sz = ctypes.c_size_t
    sig = {
        "fb_last_error": (ctypes.c_char_p, []),
        "fb_version": (ctypes.c_int32, []),
        "fb_workspace_size": (st, [P, ctypes.POINTER(sz)]),
        "fb_plan_query": (st, [P, ctypes.c_int32, ctypes.POINTER(FbPlanInfo)]),
        "fb_workspace_init": (st, [vp, sz, vp]),
        "fb_out_attn": (st, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fb_in_attn": (st, [P, vp, vp, vp, vp, vp, vp]),
        "fb_merge": (st, [ctypes.c_int64, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, vp]),
        "fb_head_similarity": (st, [P, vp, vp, vp, vp]),
        "fb_step": (st, [P, ctypes.POINTER(FbParams), ctypes.POINTER(FbCache), vp, vp, vp, vp, vp, vp, vp,
                         vp, vp, vp, vp, sz, vp]),
        "fb_cache_invalidate": (st, [P, ctypes.POINTER(FbCache), vp]),
        "fb_cache_copy_seq": (st, [P, ctypes.POINTER(FbCache), ctypes.c_int32, ctypes.c_int32, vp]),
        "fb_cache_invalidate_seqs": (st, [P, ctypes.POINTER(FbCache), vp, vp]),
        "fb_sparse_layout": (st, [P, vp, vp, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "fb_prefix_append": (st, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "fb_selftest_wait_timeout": (st, [vp]),
        "fb_release_cache": (st, []),
        "fb_device_status": (st, [ctypes.POINTER(ctypes.c_int32), vp]),
        "fb_step_noalloc": (st, [P, ctypes.POINTER(FbParams), ctypes.POINTER(FbCache), vp, vp, vp, vp, vp, vp, vp,
                                 vp, vp, vp, vp]),
        "fb_noalloc_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)  # AttributeError (loud) if the ABI is incomplete
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def last_error() -> str:
    return _lib.fb_last_error().decode()


def version() -> int:
    return int(_lib.fb_version())


def _check(status: int):
    if status != OK:
        raise FlashBlockError(status, last_error())


def _ptr(t) -> Optional[int]:
    """Device pointer of a contiguous torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------- problem / cache

class DeviceProblem:
    """A problem with its index arrays uploaded to the device (int32)."""

    def __init__(self, problem, device="cuda", out_splits: int = 0, kv_out_skip=None):
        """``kv_out_skip``: optional device uint32 bitmask over the prefix tokens (see
        fb_problem in flashblock.h); it is kept alive with the problem."""
        import torch
        self.host = problem
        self.kv_out_skip = kv_out_skip
        mk = lambda a: torch.as_tensor(np.ascontiguousarray(a, dtype=np.int32)).to(device)
        self.cu_q = mk(problem.cu_seqlens_q)
        # NULL q_rows means "row r of sequence b is block position r - cu_seqlens_q[b]"
        # (flashblock.h): passed when the active rows are exactly that
        starts = np.repeat(np.asarray(problem.cu_seqlens_q[:-1], dtype=np.int64), np.diff(problem.cu_seqlens_q))
        identity = np.array_equal(np.asarray(problem.q_rows, dtype=np.int64),
                                  np.arange(len(problem.q_rows), dtype=np.int64) - starts)
        self.q_rows = mk(problem.q_rows) if len(problem.q_rows) and not identity else None
        self.cu_out = mk(problem.cu_seqlens_kv_out)
        self.cu_in = mk(problem.cu_seqlens_kv_in)
        self.struct = FbProblem(
            problem.num_seqs, problem.num_heads_q, problem.num_heads_kv, problem.head_dim,
            float(problem.softmax_scale), _ptr(self.cu_q), _ptr(self.q_rows), _ptr(self.cu_out), _ptr(self.cu_in),
            problem.total_q, problem.total_kv_out, problem.total_kv_in,
            problem.max_q, problem.max_kv_out, problem.max_kv_in, int(out_splits), _ptr(kv_out_skip))

    @property
    def ref(self):
        return ctypes.byref(self.struct)


class Cache:
    """Caller-owned FlashBlock cache buffers (allocated with torch)."""

    def __init__(self, problem, device="cuda", with_q_ref: bool = True):
        import torch
        T, H, d = problem.total_kv_in, problem.num_heads_q, problem.head_dim
        self.a_out = torch.zeros((max(T, 1), H, d), dtype=torch.float32, device=device)
        self.l_out = torch.zeros((max(T, 1), H), dtype=torch.float32, device=device)
        self.valid = torch.zeros((max(problem.num_seqs, 1), H), dtype=torch.uint8, device=device)
        self.q_ref = torch.zeros((max(T, 1), H, d), dtype=torch.bfloat16, device=device) if with_q_ref else None
        self.m_acc = torch.zeros((max(problem.num_seqs, 1), H), dtype=torch.int32, device=device)
        self.struct = FbCache(_ptr(self.a_out), _ptr(self.l_out), _ptr(self.valid), _ptr(self.q_ref),
                              _ptr(self.m_acc))

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def params(tau: int = 0, gamma: float = 0.0, flags: int = 0) -> FbParams:
    return FbParams(int(tau), float(gamma), int(flags))


# ---------------------------------------------------------------- calls

def plan_query(problem: DeviceProblem, call: int = CALL_STEP) -> dict:
    """fb_plan_query: the launch plan of a call as a dict (plus ``kernel_name``).
    Host computation only; the problem's index arrays may live on the host."""
    info = FbPlanInfo()
    _check(_lib.fb_plan_query(problem.ref, int(call), ctypes.byref(info)))
    out = {name: int(getattr(info, name)) for name, _ in FbPlanInfo._fields_}
    out["kernel_name"] = KERNEL_NAMES[out["kernel"]]
    return out


def workspace_size(problem: DeviceProblem) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.fb_workspace_size(problem.ref, ctypes.byref(n)))
    return int(n.value)


def workspace_init(workspace, stream=None):
    _check(_lib.fb_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def alloc_workspace(problem: DeviceProblem, device="cuda"):
    import torch
    ws = torch.empty(max(workspace_size(problem), 16), dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def out_attn(problem: DeviceProblem, q, k_out, v_out, a_out, l_out, workspace, head_mask=None, stream=None):
    _check(_lib.fb_out_attn(problem.ref, _ptr(q), _ptr(k_out), _ptr(v_out), _ptr(head_mask), _ptr(a_out),
                            _ptr(l_out), _ptr(workspace), workspace.numel(), _stream(stream)))


def in_attn(problem: DeviceProblem, q, k_in, v_in, a_in, l_in, stream=None):
    _check(_lib.fb_in_attn(problem.ref, _ptr(q), _ptr(k_in), _ptr(v_in), _ptr(a_in), _ptr(l_in), _stream(stream)))


def merge(a_out, l_out, a_in, l_in, a_full_f32=None, a_full_bf16=None, l_full=None, stream=None):
    n = l_out.numel()
    d = a_out.numel() // max(n, 1)
    _check(_lib.fb_merge(n, d, _ptr(a_out), _ptr(l_out), _ptr(a_in), _ptr(l_in), _ptr(a_full_f32),
                         _ptr(a_full_bf16), _ptr(l_full), _stream(stream)))


def head_similarity(problem: DeviceProblem, q, q_ref, cos_out, stream=None):
    _check(_lib.fb_head_similarity(problem.ref, _ptr(q), _ptr(q_ref), _ptr(cos_out), _stream(stream)))


def step(problem: DeviceProblem, prm: FbParams, cache: Cache, q, k_in, v_in, k_out, v_out, n_updated,
         a_full, workspace, l_full=None, head_reuse_in=None, decision_out=None, stream=None):
    _check(_lib.fb_step(problem.ref, ctypes.byref(prm), cache.ref, _ptr(q), _ptr(k_in), _ptr(v_in), _ptr(k_out),
                        _ptr(v_out), _ptr(n_updated), _ptr(head_reuse_in), _ptr(a_full), _ptr(l_full),
                        _ptr(decision_out), _ptr(workspace), workspace.numel(), _stream(stream)))


def step_noalloc(problem: DeviceProblem, prm: FbParams, cache: Cache, q, k_in, v_in, k_out, v_out, n_updated,
                 a_full, l_full=None, head_reuse_in=None, decision_out=None, stream=None):
    """fb_step without a workspace: for callers that cannot allocate device memory,
    the library uses its own built-in scratch (see fb_step_noalloc in flashblock.h)."""
    status = _lib.fb_step_noalloc(problem.ref, ctypes.byref(prm), cache.ref, _ptr(q), _ptr(k_in), _ptr(v_in),
                                  _ptr(k_out), _ptr(v_out), _ptr(n_updated), _ptr(head_reuse_in), _ptr(a_full),
                                  _ptr(l_full), _ptr(decision_out), _stream(stream))
    if status != OK:
        msg = _lib.fb_noalloc_last_error().decode() or last_error()
        raise FlashBlockError(status, msg)


def cache_invalidate(problem: DeviceProblem, cache: Cache, stream=None):
    _check(_lib.fb_cache_invalidate(problem.ref, cache.ref, _stream(stream)))


def cache_copy_seq(problem: DeviceProblem, cache: Cache, src_seq: int, dst_seq: int, stream=None):
    _check(_lib.fb_cache_copy_seq(problem.ref, cache.ref, int(src_seq), int(dst_seq), _stream(stream)))


def cache_invalidate_seqs(problem: DeviceProblem, cache: Cache, seq_mask=None, stream=None):
    _check(_lib.fb_cache_invalidate_seqs(problem.ref, cache.ref, _ptr(seq_mask), _stream(stream)))


def sparse_layout(problem: DeviceProblem, cu_sel, sel_idx, total_sel: int, k_out, v_out, k_in, v_in,
                  k_ext, v_ext, kv_out_skip, cu_in_ext=None, stream=None):
    """fb_sparse_layout: selected prefix keys join the block's keys (k_ext, v_ext) and are
    marked in the prefix skip mask (see flashblock.h)."""
    _check(_lib.fb_sparse_layout(problem.ref, _ptr(cu_sel), _ptr(sel_idx), int(total_sel), _ptr(k_out), _ptr(v_out),
                                 _ptr(k_in), _ptr(v_in), _ptr(k_ext), _ptr(v_ext), _ptr(kv_out_skip),
                                 _ptr(cu_in_ext), _stream(stream)))


def prefix_append(problem: DeviceProblem, k_out, v_out, k_in, v_in, k_dst, v_dst, cu_out_dst=None, stream=None):
    """fb_prefix_append: block transition -- each sequence's finished block K/V follow
    its prefix in (k_dst, v_dst) (see flashblock.h)."""
    _check(_lib.fb_prefix_append(problem.ref, _ptr(k_out), _ptr(v_out), _ptr(k_in), _ptr(v_in), _ptr(k_dst),
                                 _ptr(v_dst), _ptr(cu_out_dst), _stream(stream)))


def selftest_wait_timeout(stream=None):
    _check(_lib.fb_selftest_wait_timeout(_stream(stream)))


def release_cache():
    _check(_lib.fb_release_cache())


def device_status(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(_lib.fb_device_status(ctypes.byref(code), _stream(stream)))
    return int(code.value)


def bf16_tensor(bits: np.ndarray, device="cuda"):
    """Upload bf16 bit patterns (numpy uint16) as a torch.bfloat16 tensor."""
    import torch
    a = np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(a).to(device).view(torch.bfloat16)
