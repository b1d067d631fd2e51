// fb_step_noalloc: fb_step for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: code that runs where a
// cudaMalloc is not allowed or not wanted (inside a framework whose allocator
// owns all device memory, in a plugin that must not allocate, in a
// latency-critical loop where an allocation would synchronise the device).  For
// them this entry point uses a scratch array that lives in the library itself: a
// file-scope __device__ array of fixed size that every GPU loading the library
// holds until the process exits.  Nothing is allocated at call time.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "flashblock.h"

namespace {

// Scratch of every call: a call runs when its fb_workspace_size fits here -- a
// 256-byte completion-counter slot plus one fp32 similarity score per (sequence,
// q-head), i.e. up to 16320 such pairs, fewer when the workspace also holds the
// two-tile kernel's work order (one int32 per (sequence, head, 256-row pair)).
constexpr size_t kScratchBytes = 64 * 1024;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

thread_local char t_msg[512];

void set_msg(const char* fmt, const char* a, const char* b = "") { snprintf(t_msg, sizeof(t_msg), fmt, a, b); }

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 when the driver cannot tell).  A device's
// primary context gets a new id when it is re-created (after cudaDeviceReset), and
// the scratch array then has a new address.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {  // under g_mu
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
    cudaGetLastError();
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

// Device address of the scratch array on the current device (host code only sees
// a host-side stand-in under the array's name).  Resolved with the device current
// on the first call of each device, and again only if that device's context was
// re-created since.
fb_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_msg("fb_step_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return FB_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(t_msg, sizeof(t_msg), "fb_step_noalloc: device ordinal %d is above %d", dev, kMaxDevices - 1);
    return FB_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  const unsigned long long ctx = current_ctx_id();
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      set_msg("fb_step_noalloc: cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      return FB_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return FB_OK;
}

}  // namespace

extern "C" {

const char* fb_noalloc_last_error(void) { return t_msg; }

fb_status fb_step_noalloc(const fb_problem* problem, const fb_params* params, const fb_cache* cache,
                          const fb_bf16* q, const fb_bf16* k_in, const fb_bf16* v_in, const fb_bf16* k_out,
                          const fb_bf16* v_out, const int32_t* n_updated, const uint8_t* head_reuse_in,
                          fb_bf16* a_full, float* l_full, uint8_t* decision_out, fb_stream_t stream) {
  t_msg[0] = 0;
  size_t need = 0;
  fb_status st = fb_workspace_size(problem, &need);
  if (st != FB_OK) {  // argument errors
    set_msg("fb_step_noalloc: %s", fb_last_error());
    return st;
  }
  if (need > kScratchBytes) {
    snprintf(t_msg, sizeof(t_msg),
             "fb_step_noalloc: this problem needs %zu bytes of scratch, above the built-in %zu bytes "
             "(num_seqs x num_heads_q too large); use fb_step with a workspace",
             need, kScratchBytes);
    return FB_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != FB_OK) return st;
  // The completion counter must read zero when the kernel starts.
  cudaError_t e = cudaMemsetAsync(scratch, 0, 256, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_msg("fb_step_noalloc: cudaMemsetAsync(scratch counter): %s", cudaGetErrorString(e));
    return FB_ERR_CUDA;
  }
  st = fb_step(problem, params, cache, q, k_in, v_in, k_out, v_out, n_updated, head_reuse_in, a_full, l_full,
               decision_out, scratch, kScratchBytes, stream);
  if (st != FB_OK) set_msg("fb_step_noalloc: %s", fb_last_error());
  return st;
}

}  // extern "C"
