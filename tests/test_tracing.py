"""NVTX ranges of the C ABI (CPU).

A small NVTX injection library, built here with gcc and handed to NVTX through
NVTX_INJECTION64_PATH in a child process, records the ranges the library's entry
points push and pop.  Every call below fails a host-side argument check before any
CUDA call, so no GPU is needed; the range must be closed on that early return too."""
import json
import os
import shutil
import subprocess
import sys

import pytest

# Records each pushed range's name and the push/pop balance.  The callback slots and
# their ids are the ones NVTX's public export-table interface defines.
INJECTION_C = r"""
#include <string.h>
#include <nvtx3/nvToolsExt.h>

#define MAX_RANGES 256
static char g_names[MAX_RANGES][48];
static int g_pushes, g_pops, g_depth, g_max_depth, g_underflow;

static int on_push(const char* msg) {
  if (g_pushes < MAX_RANGES) {
    strncpy(g_names[g_pushes], msg ? msg : "", sizeof(g_names[0]) - 1);
  }
  ++g_pushes;
  if (++g_depth > g_max_depth) g_max_depth = g_depth;
  return g_depth - 1;
}

static int on_pop(void) {
  ++g_pops;
  if (--g_depth < 0) { g_underflow = 1; g_depth = 0; }
  return g_depth;
}

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size)) return 0;
  if (size <= NVTX_CBID_CORE_RangePop) return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)on_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)on_pop;
  return 1;
}

int rec_pushes(void) { return g_pushes; }
int rec_pops(void) { return g_pops; }
int rec_depth(void) { return g_depth; }
int rec_max_depth(void) { return g_max_depth; }
int rec_underflow(void) { return g_underflow; }
const char* rec_name(int i) { return (i >= 0 && i < MAX_RANGES) ? g_names[i] : ""; }
"""

# Runs in the child: each entry point once with arguments its host checks reject,
# then the recorder's view as one JSON line.
CHILD = r"""
import ctypes, json, sys
lib = ctypes.CDLL(sys.argv[1])
rec = ctypes.CDLL(sys.argv[2])
rec.rec_name.restype = ctypes.c_char_p
N = None
calls = [
    ("fb_workspace_init", lambda: lib.fb_workspace_init(N, ctypes.c_size_t(16), N)),
    ("fb_out_attn", lambda: lib.fb_out_attn(*([N] * 8), ctypes.c_size_t(0), N)),
    ("fb_in_attn", lambda: lib.fb_in_attn(*([N] * 7))),
    ("fb_merge", lambda: lib.fb_merge(ctypes.c_int64(1), ctypes.c_int32(128), *([N] * 8))),
    ("fb_head_similarity", lambda: lib.fb_head_similarity(*([N] * 5))),
    ("fb_step", lambda: lib.fb_step(*([N] * 14), ctypes.c_size_t(0), N)),
    ("fb_cache_invalidate", lambda: lib.fb_cache_invalidate(N, N, N)),
    ("fb_cache_copy_seq", lambda: lib.fb_cache_copy_seq(N, N, ctypes.c_int32(0), ctypes.c_int32(1), N)),
    ("fb_cache_invalidate_seqs", lambda: lib.fb_cache_invalidate_seqs(N, N, N, N)),
    ("fb_sparse_layout", lambda: lib.fb_sparse_layout(N, N, N, ctypes.c_int32(0), *([N] * 9))),
    ("fb_prefix_append", lambda: lib.fb_prefix_append(*([N] * 9))),
    ("fb_device_status", lambda: lib.fb_device_status(N, N)),
]
status = {}
for name, call in calls:
    status[name] = call()
# calls that enqueue nothing open no range
size = ctypes.c_size_t()
quiet = [lib.fb_workspace_size(N, ctypes.byref(size)), lib.fb_plan_query(N, ctypes.c_int32(0), N),
         lib.fb_version(), lib.fb_release_cache()]
n = rec.rec_pushes()
print(json.dumps(dict(status=status, quiet=quiet, names=[rec.rec_name(i).decode() for i in range(n)],
                      pushes=n, pops=rec.rec_pops(), depth=rec.rec_depth(), max_depth=rec.rec_max_depth(),
                      underflow=rec.rec_underflow())))
"""


def _cuda_include():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "include")
    return inc if os.path.exists(os.path.join(inc, "nvtx3", "nvToolsExt.h")) else None


def test_every_enqueuing_call_opens_and_closes_its_range(tmp_path):
    gcc = shutil.which("gcc")
    inc = _cuda_include()
    if gcc is None or inc is None:
        pytest.skip("gcc or the NVTX headers are not available")
    from cached_split_attention_b200 import build
    lib = build.build()
    src = tmp_path / "nvtx_recorder.c"
    src.write_text(INJECTION_C)
    so = str(tmp_path / "libnvtx_recorder.so")
    r = subprocess.run([gcc, "-std=gnu11", "-O1", "-fPIC", "-shared", "-I", inc, str(src), "-o", so],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, NVTX_INJECTION64_PATH=so, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", CHILD, lib, so], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    # every call was rejected by its host checks (FB_ERR_INVALID_ARG = 1)
    assert all(v == 1 for v in out["status"].values()), out["status"]
    # one range per call, named for it, in call order, each closed on the early return
    assert out["names"] == list(out["status"].keys())
    assert out["pushes"] == out["pops"] == len(out["status"])
    assert out["depth"] == 0 and out["max_depth"] == 1 and not out["underflow"]
    # the query calls opened none
    assert out["quiet"][0] == 1 and out["quiet"][1] == 1 and out["quiet"][3] == 0


def test_without_a_tool_the_ranges_do_nothing():
    """No injection: the library's calls behave exactly as before (same status)."""
    from cached_split_attention_b200 import build
    lib = build.build()
    env = {k: v for k, v in os.environ.items() if k != "NVTX_INJECTION64_PATH"}
    code = ("import ctypes, sys; lib = ctypes.CDLL(sys.argv[1]); "
            "print(lib.fb_step(*([None] * 14), ctypes.c_size_t(0), None), lib.fb_device_status(None, None))")
    r = subprocess.run([sys.executable, "-c", code, lib], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.split() == ["1", "1"]
