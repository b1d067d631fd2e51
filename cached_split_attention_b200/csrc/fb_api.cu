// Host side of the C ABI declared in include/flashblock.h: argument checks,
// launch planning, the TMA descriptor cache and the kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "fb_order.cuh"
#include "fb_selftest.cuh"
#include "fb_sparse.cuh"
#include "fb_tc2_kernel.cuh"
#include "fb_transition.cuh"
#include "flashblock.h"

namespace {

thread_local std::string t_err = "no error";

// An NVTX range around one call that enqueues device work, named for the entry
// point, so that a timeline tool shows where each call's launches were issued.
// NVTX does nothing unless a tool is attached to the process.
class Range {
 public:
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

fb_status fail(fb_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

fb_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FB_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ validation

fb_status check_problem(const fb_problem* p) {
  if (!p) return fail(FB_ERR_INVALID_ARG, "problem is NULL");
  if (p->num_seqs < 0) return fail(FB_ERR_INVALID_ARG, "num_seqs < 0");
  if (p->num_heads_q <= 0 || p->num_heads_kv <= 0) return fail(FB_ERR_INVALID_ARG, "head counts must be > 0");
  if (p->num_heads_q % p->num_heads_kv != 0)
    return fail(FB_ERR_UNSUPPORTED, "num_heads_q (%d) is not a multiple of num_heads_kv (%d)", p->num_heads_q,
                p->num_heads_kv);
  if (p->num_heads_q / p->num_heads_kv > fb::kMaxGroup)
    return fail(FB_ERR_UNSUPPORTED, "query heads per kv head > %d", fb::kMaxGroup);
  if (p->head_dim != 64 && p->head_dim != 128) return fail(FB_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", p->head_dim);
  if (!(p->softmax_scale > 0.f) || !std::isfinite(p->softmax_scale))
    return fail(FB_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (p->total_q < 0 || p->total_kv_out < 0 || p->total_kv_in < 0 || p->max_q < 0 || p->max_kv_out < 0 ||
      p->max_kv_in < 0)
    return fail(FB_ERR_INVALID_ARG, "negative size");
  if (p->max_q > p->total_q || p->max_kv_out > p->total_kv_out || p->max_kv_in > p->total_kv_in)
    return fail(FB_ERR_INVALID_ARG, "a per-sequence maximum exceeds its total");
  if (p->max_q > p->max_kv_in) return fail(FB_ERR_INVALID_ARG, "max_q exceeds max_kv_in (rows are block positions)");
  if (p->out_splits < 0) return fail(FB_ERR_INVALID_ARG, "out_splits < 0");
  if (static_cast<int64_t>(p->total_kv_in) * p->num_heads_q >= (int64_t{1} << 31) ||
      static_cast<int64_t>(p->total_q) * p->num_heads_q >= (int64_t{1} << 31))
    return fail(FB_ERR_UNSUPPORTED, "tokens x query heads must stay below 2^31");
  // The grid has up to num_seqs x num_heads_q x max_q x kMaxSplits CTAs (every
  // sequence is sized by the longest); keep it, and the per-(sequence, head)
  // workspace arrays, inside 32-bit indices.
  if (static_cast<int64_t>(p->num_seqs) * p->num_heads_q * std::max(1, p->max_q) * fb::kMaxSplits >=
      (int64_t{1} << 31))
    return fail(FB_ERR_UNSUPPORTED, "num_seqs x num_heads_q x max_q is too large for one launch");
  if (p->num_seqs > 0 && (!p->cu_seqlens_q || !p->cu_seqlens_kv_out || !p->cu_seqlens_kv_in))
    return fail(FB_ERR_INVALID_ARG, "cu_seqlens arrays must not be NULL");
  if (p->kv_out_skip && (reinterpret_cast<uintptr_t>(p->kv_out_skip) & 3u))
    return fail(FB_ERR_INVALID_ARG, "kv_out_skip is not 4-byte aligned");
  return FB_OK;
}

fb_status check_ptr(const void* ptr, const char* name, bool needed) {
  if (!needed) return FB_OK;
  if (!ptr) return fail(FB_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(ptr)) return fail(FB_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return FB_OK;
}

#define FB_TRY(x)                     \
  do {                                \
    fb_status _s = (x);               \
    if (_s != FB_OK) return _s;       \
  } while (0)

// ------------------------------------------------------------------ planning

struct Plan {
  int d = 0, g = 0, wm = 0, tr = 0, tiles = 0, n_groups = 0, splits = 1, threads = 0, smem = 0;
  bool tc = false;   // tensor-core kernel (tcgen05): head_dim 128, more than 64 rows per group
  bool tc2 = false;  // two-tile tensor-core kernel: fused step, MHA, at least 256 rows per head
  bool tc_split = false;  // tensor-core kernel with two threads per tile row (grids of more than one wave)
  int bn = fb::kBN;  // keys per pipeline chunk (TMA box rows)
  size_t off_grid_ctr = 0, off_cos = 0, off_order = 0, bytes = 0;
  int order_items = 0;  // work items of the two-tile kernel (0: the problem never takes it)
  // lean reuse path (fused step, blocks of at most reuse::kMaxKeys keys)
  bool reuse = false;
  int reuse_chunks = 0, reuse_smem = 0, reuse_bt = 0;
  bool reuse_early = false;  // every CTA resident at once: lean loads before the decision
};

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Tile shapes: WM row slabs of 16 rows x WN key shares = 8 warps per CTA (4 for
// 16-row tiles), one CTA per SM; stage ring of 128 KB (96 KB for 128-row tiles).
struct Shape {
  void* fn;
  int threads;
  int smem;
};

template <int D, int WM>
Shape shape_of() {
  constexpr int WN = WM == 1 ? 4 : 8 / WM;
  constexpr int ST = (D == 64 ? 2 : 1) * (WM == 8 ? 3 : 4);
  using C = fb::Cfg<D, WM, WN, ST>;
  return {reinterpret_cast<void*>(&fb::attn_kernel<D, WM, WN, ST>), C::kThreads, C::kSmem};
}

Shape shape_for(int d, int wm) {
  if (d == 64) {
    switch (wm) {
      case 1: return shape_of<64, 1>();
      case 2: return shape_of<64, 2>();
      case 4: return shape_of<64, 4>();
      default: return shape_of<64, 8>();
    }
  }
  // head_dim 128: groups of more than 64 rows (WM = 8) take the tensor-core kernel
  switch (wm) {
    case 1: return shape_of<128, 1>();
    case 2: return shape_of<128, 2>();
    default: return shape_of<128, 4>();
  }
}

// in_only: fb_in_attn (no prefix pass, one CTA per group)
// Groups of at least this many rows (head_dim 128) go to the tensor-core kernel.
constexpr int kTcMinRows = 65;

Plan make_plan(const fb_problem* p, int num_sms, bool in_only, bool fused = false) {
  Plan pl;
  pl.d = p->head_dim;
  pl.g = p->num_heads_q / p->num_heads_kv;
  const long rows = static_cast<long>(pl.g) * p->max_q;
  pl.wm = rows <= 16 ? 1 : rows <= 32 ? 2 : rows <= 64 ? 4 : 8;
  pl.tc = pl.d == 128 && rows >= kTcMinRows;
  pl.tc2 = fused && pl.d == 128 && pl.g == 1 && p->max_q >= 2 * fb::tc2::kM;
  if (pl.tc2) {
    pl.threads = fb::tc2::kThreads;
    pl.smem = fb::tc2::kSmem;
    pl.tr = 2 * fb::tc2::kM;
    pl.bn = fb::tc2::kN;
  } else if (pl.tc) {
    pl.threads = fb::tc::threads_for(1);
    pl.smem = fb::tc::kSmem;
    pl.tr = fb::tc::kM;
    pl.bn = fb::tc::kN;
  } else {
    const Shape sh = shape_for(pl.d, pl.wm);
    pl.threads = sh.threads;
    pl.smem = sh.smem;
    pl.tr = 16 * pl.wm;
    pl.bn = fb::kBN;
  }
  pl.tiles = static_cast<int>(std::max<long>(1, (rows + pl.tr - 1) / pl.tr));
  pl.n_groups = p->num_seqs * p->num_heads_kv * pl.tiles;
  const int chunks = std::max(1, (p->max_kv_out + pl.bn - 1) / pl.bn);
  int splits = 1;
  if (!in_only && !pl.tc2) {
    if (p->out_splits > 0) {
      splits = p->out_splits;
    } else {
      // One wave: as many CTAs per group as the resident slots allow.  (A split
      // chosen by makespan -- more waves of shorter CTAs -- was measured slower:
      // the per-CTA lead-in and merge outweigh the better packing of the waves.)
      const int per_sm = std::max(1, std::min(233472 / (pl.smem + 1024), 2048 / pl.threads));
      const long slots = static_cast<long>(num_sms) * per_sm;
      splits = static_cast<int>(std::max(1L, slots / std::max(1, pl.n_groups)));
    }
    splits = std::max(1, std::min({splits, fb::kMaxSplits, chunks}));
  }
  pl.splits = splits;
  // More CTAs than one wave holds (the varlen branches): the later CTAs run with the
  // HBM less loaded, where one softmax thread per row bounds the stream; two threads
  // per row (twice the softmax warps) suit them.  A full single wave is bound by HBM,
  // and there the extra per-chunk exchange of the two halves costs a little.
  if (pl.tc && !pl.tc2) {
    const int per_sm = std::max(1, std::min(233472 / (pl.smem + 1024), 2048 / pl.threads));
    if (static_cast<long>(pl.n_groups) * pl.splits > static_cast<long>(num_sms) * per_sm) {
      pl.tc_split = true;
      pl.threads = fb::tc::threads_for(2);
    }
  }
  // Lean reuse path: blocks of up to 128 keys, when the kernel's shared memory
  // holds the block K/V and a tile of rows with their cache entries.
  if (fused && !pl.tc2 && p->max_kv_in > 0 && p->max_kv_in <= fb::reuse::kMaxKeys && rows > 0) {
    const int chunks = (p->max_kv_in + fb::kBN - 1) / fb::kBN;
    // most rows a CTA takes (lean_rows: whole 16-row slabs shared by the splits)
    const int slabs = static_cast<int>((std::min<long>(pl.tr, rows) + 15) / 16);
    const int nr_max = (slabs + pl.splits - 1) / pl.splits * 16;
    const int bt = fb::reuse::box_tokens(pl.g, nr_max);
    const int need = fb::reuse::smem_bytes(pl.d, chunks, pl.g, bt) + 1024;
    // TMA box extents are at most 256; a box token's thread is one of warps 1..
    if (need <= pl.smem && pl.g <= 256 && bt <= 256 && bt <= pl.threads - fb::kLeanTok0) {
      const int per_sm = std::max(1, std::min(233472 / (pl.smem + 1024), 2048 / pl.threads));
      pl.reuse = true;
      pl.reuse_chunks = chunks;
      pl.reuse_smem = need;
      pl.reuse_bt = bt;
      pl.reuse_early = static_cast<long>(pl.n_groups) * pl.splits <= static_cast<long>(num_sms) * per_sm;
    }
  }
  // workspace layout
  size_t off = 0;
  pl.off_grid_ctr = off;
  off = align_up(off + sizeof(int), 256);
  pl.off_cos = off;
  off = align_up(off + sizeof(float) * std::max(1, p->num_seqs * p->num_heads_q), 256);
  // work order of the two-tile kernel, for every problem that fb_step may give it
  if (pl.d == 128 && pl.g == 1 && p->max_q >= 2 * fb::tc2::kM) {
    pl.order_items = p->num_seqs * p->num_heads_q * ((p->max_q + 2 * fb::tc2::kM - 1) / (2 * fb::tc2::kM));
    pl.off_order = off;
    off = align_up(off + sizeof(int) * pl.order_items, 256);
  }
  pl.bytes = off;
  return pl;
}

// ------------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_map_mu;
std::unordered_map<std::string, CUtensorMap> g_maps;
EncodeTiledFn g_encode = nullptr;

fb_status get_encode(EncodeTiledFn* fn) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (!g_encode) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f)
      return fail(FB_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    g_encode = reinterpret_cast<EncodeTiledFn>(f);
  }
  *fn = g_encode;
  return FB_OK;
}

// Map of a THD bf16 buffer [tokens, hkv, d] viewed as 2-D {hkv*d, tokens}; the box
// is 64 columns (128 bytes, the swizzle span) by kBN token rows.
fb_status kv_map(const void* ptr, int tokens, int hkv, int d, int box_rows, CUtensorMap* out) {
  std::memset(out, 0, sizeof(*out));
  if (tokens <= 0) return FB_OK;  // never read: every key range is empty
  int dev = 0;
  cudaGetDevice(&dev);
  char key[96];
  snprintf(key, sizeof(key), "%d:%p:%d:%d:%d:%d", dev, ptr, tokens, hkv, d, box_rows);
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return FB_OK;
    }
  }
  EncodeTiledFn enc;
  FB_TRY(get_encode(&enc));
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(hkv) * d, static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(hkv) * d * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FB_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, *out);
  return FB_OK;
}

// Map of the packed queries [tokens, hq, d] bf16 as 3-D {d, hq, tokens}; the box is
// 64 columns (the swizzle span) x g heads x bt tokens: a lean CTA's Q rows.
fb_status q_map(const void* ptr, int tokens, int hq, int d, int g, int bt, CUtensorMap* out) {
  std::memset(out, 0, sizeof(*out));
  if (tokens <= 0) return FB_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  char key[112];
  snprintf(key, sizeof(key), "q%d:%p:%d:%d:%d:%d:%d", dev, ptr, tokens, hq, d, g, bt);
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return FB_OK;
    }
  }
  EncodeTiledFn enc;
  FB_TRY(get_encode(&enc));
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(hq), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(hq) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(bt)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FB_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, *out);
  return FB_OK;
}

// ------------------------------------------------------------------ launch

fb_status launch_attn(const Plan& pl, fb::Params& prm, cudaStream_t stream) {
  const int n_ctas = pl.n_groups * pl.splits;
  if (n_ctas <= 0) return FB_OK;
  void* fn = pl.tc2  ? reinterpret_cast<void*>(&fb::tc2_attn_kernel)
             : pl.tc ? (pl.tc_split ? reinterpret_cast<void*>(&fb::tc_attn_kernel<2>)
                                    : reinterpret_cast<void*>(&fb::tc_attn_kernel<1>))
                     : shape_for(pl.d, pl.wm).fn;
  static std::mutex mu;
  static bool attr_done[5][9] = {};
  {
    std::lock_guard<std::mutex> lk(mu);
    bool& done = attr_done[pl.tc2 ? 3 : pl.tc ? (pl.tc_split ? 4 : 2) : (pl.d == 128)][pl.wm];
    if (!done) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      done = true;
    }
  }
  prm.splits = pl.splits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pl.splits > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = pl.splits;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  void* args[] = {&prm};
  cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return FB_OK;
}

// Launch of a kernel without clusters, allowed to start while the previous
// kernel of the stream finishes (each kernel waits for it before reading).
template <typename... Args>
cudaError_t launch_pdl(void (*fn)(Args...), int blocks, int threads, cudaStream_t stream, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* argv[] = {const_cast<void*>(static_cast<const void*>(&args))...};  // copied at launch
  return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(fn), argv);
}

void fill_problem(const fb_problem* p, const Plan& pl, fb::Params& prm) {
  prm.num_seqs = p->num_seqs;
  prm.hq = p->num_heads_q;
  prm.hkv = p->num_heads_kv;
  prm.g = pl.g;
  prm.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  prm.cu_q = p->cu_seqlens_q;
  prm.q_rows = p->q_rows;
  prm.cu_out = p->cu_seqlens_kv_out;
  prm.cu_in = p->cu_seqlens_kv_in;
  prm.total_q = p->total_q;
  prm.total_out = p->total_kv_out;
  prm.total_in = p->total_kv_in;
  prm.tiles = pl.tiles;
  prm.splits = pl.splits;
  prm.out_skip = p->kv_out_skip;
}

void fill_workspace(const Plan& pl, void* ws, fb::Params& prm) {
  char* base = static_cast<char*>(ws);
  prm.grid_ctr = reinterpret_cast<int*>(base + pl.off_grid_ctr);
  prm.cos = reinterpret_cast<const float*>(base + pl.off_cos);
}

}  // namespace

// ==================================================================== C ABI

extern "C" {

const char* fb_last_error(void) { return t_err.c_str(); }

int32_t fb_version(void) { return 100; }

fb_status fb_plan_query(const fb_problem* problem, int32_t call, fb_plan_info* out) {
  FB_TRY(check_problem(problem));
  if (!out) return fail(FB_ERR_INVALID_ARG, "out is NULL");
  if (call != FB_CALL_STEP && call != FB_CALL_OUT && call != FB_CALL_IN)
    return fail(FB_ERR_INVALID_ARG, "unknown call %d", call);
  const int sms = device_sms();
  const Plan pl = make_plan(problem, sms, call == FB_CALL_IN, call == FB_CALL_STEP);
  out->kernel = pl.tc2 ? FB_KERNEL_TC2 : pl.tc ? FB_KERNEL_TC : FB_KERNEL_WARP_MMA;
  out->rows_per_tile = pl.tc2 ? pl.tr / 2 : pl.tr;
  const long rows = static_cast<long>(pl.g) * problem->max_q;
  out->tiles = pl.tc2 ? static_cast<int>(std::max<long>(1, (rows + pl.tr / 2 - 1) / (pl.tr / 2))) : pl.tiles;
  out->work_items = pl.n_groups;
  out->splits = pl.splits;
  out->ctas = pl.n_groups * pl.splits;
  out->threads = pl.threads;
  out->smem_bytes = pl.smem;
  out->keys_per_chunk = pl.bn;
  out->num_sms = sms;
  out->lean_reuse = pl.reuse ? 1 : 0;
  out->lean_smem_bytes = pl.reuse ? pl.reuse_smem : 0;
  out->lean_early = pl.reuse && pl.reuse_early ? 1 : 0;
  return FB_OK;
}

fb_status fb_workspace_size(const fb_problem* problem, size_t* bytes) {
  FB_TRY(check_problem(problem));
  if (!bytes) return fail(FB_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = make_plan(problem, device_sms(), false).bytes;
  return FB_OK;
}

fb_status fb_workspace_init(void* workspace, size_t bytes, fb_stream_t stream) {
  const Range range("fb_workspace_init");
  if (!workspace && bytes) return fail(FB_ERR_INVALID_ARG, "workspace is NULL");
  if (!bytes) return FB_OK;
  cudaError_t e = cudaMemsetAsync(workspace, 0, bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
  return FB_OK;
}

fb_status fb_out_attn(const fb_problem* problem, const fb_bf16* q, const fb_bf16* k_out, const fb_bf16* v_out,
                      const uint8_t* head_mask, float* a_out, float* l_out, void* workspace, size_t workspace_bytes,
                      fb_stream_t stream) {
  const Range range("fb_out_attn");
  FB_TRY(check_problem(problem));
  const bool rows = problem->total_q > 0;
  FB_TRY(check_ptr(q, "q", rows));
  FB_TRY(check_ptr(k_out, "k_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(v_out, "v_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(a_out, "a_out", rows));
  if (rows && !l_out) return fail(FB_ERR_INVALID_ARG, "l_out is NULL");
  if (problem->num_seqs == 0 || !rows) return FB_OK;
  const Plan pl = make_plan(problem, device_sms(), false);
  if (!workspace || workspace_bytes < pl.bytes)
    return fail(FB_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, pl.bytes);
  fb::Params prm;
  std::memset(&prm, 0, sizeof(prm));
  fill_problem(problem, pl, prm);
  fill_workspace(pl, workspace, prm);
  FB_TRY(kv_map(k_out, problem->total_kv_out, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_k_out));
  FB_TRY(kv_map(v_out, problem->total_kv_out, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_v_out));
  prm.q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm.do_out = 1;
  prm.head_mask = head_mask;
  prm.cache_a = a_out;
  prm.cache_l = l_out;
  return launch_attn(pl, prm, reinterpret_cast<cudaStream_t>(stream));
}

fb_status fb_in_attn(const fb_problem* problem, const fb_bf16* q, const fb_bf16* k_in, const fb_bf16* v_in,
                     float* a_in, float* l_in, fb_stream_t stream) {
  const Range range("fb_in_attn");
  FB_TRY(check_problem(problem));
  const bool rows = problem->total_q > 0;
  FB_TRY(check_ptr(q, "q", rows));
  FB_TRY(check_ptr(k_in, "k_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(v_in, "v_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(a_in, "a_in", rows));
  if (rows && !l_in) return fail(FB_ERR_INVALID_ARG, "l_in is NULL");
  if (problem->num_seqs == 0 || !rows) return FB_OK;
  const Plan pl = make_plan(problem, device_sms(), true);
  fb::Params prm;
  std::memset(&prm, 0, sizeof(prm));
  fill_problem(problem, pl, prm);
  FB_TRY(kv_map(k_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_k_in));
  FB_TRY(kv_map(v_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_v_in));
  prm.q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm.do_in = 1;
  prm.a_in = a_in;
  prm.l_in = l_in;
  return launch_attn(pl, prm, reinterpret_cast<cudaStream_t>(stream));
}

fb_status fb_merge(int64_t n, int32_t d, const float* a_out, const float* l_out, const float* a_in,
                   const float* l_in, float* a_full_f32, fb_bf16* a_full_bf16, float* l_full, fb_stream_t stream) {
  const Range range("fb_merge");
  if (n < 0 || d <= 0) return fail(FB_ERR_INVALID_ARG, "n must be >= 0 and d > 0");
  if (n > INT64_MAX / d) return fail(FB_ERR_INVALID_ARG, "n x d overflows 64 bits");
  if (n == 0) return FB_OK;
  if (!a_out || !l_out || !a_in || !l_in) return fail(FB_ERR_INVALID_ARG, "merge inputs must not be NULL");
  if (!a_full_f32 && !a_full_bf16) return fail(FB_ERR_INVALID_ARG, "no output for A_full");
  fb::MergeParams mp{n, d, a_out, l_out, a_in, l_in, a_full_f32, reinterpret_cast<__nv_bfloat16*>(a_full_bf16),
                     l_full};
  const int64_t total = n * static_cast<int64_t>(d);
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 16));
  cudaError_t e = launch_pdl(fb::merge_kernel, blocks, 256, reinterpret_cast<cudaStream_t>(stream), mp);
  if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
  return FB_OK;
}

fb_status fb_head_similarity(const fb_problem* problem, const fb_bf16* q, const fb_bf16* q_ref, float* cos_out,
                             fb_stream_t stream) {
  const Range range("fb_head_similarity");
  FB_TRY(check_problem(problem));
  FB_TRY(check_ptr(q, "q", problem->total_q > 0));
  FB_TRY(check_ptr(q_ref, "q_ref", problem->total_kv_in > 0));
  if (!cos_out && problem->num_seqs > 0) return fail(FB_ERR_INVALID_ARG, "cos_out is NULL");
  if (problem->num_seqs == 0) return FB_OK;
  fb::SimParams sp{problem->num_heads_q, problem->head_dim, problem->total_q, problem->total_kv_in,
                   problem->cu_seqlens_q, problem->q_rows,
                   problem->cu_seqlens_kv_in, reinterpret_cast<const __nv_bfloat16*>(q),
                   reinterpret_cast<const __nv_bfloat16*>(q_ref), cos_out};
  cudaError_t e = launch_pdl(fb::similarity_kernel, problem->num_seqs * problem->num_heads_q, 256,
                             reinterpret_cast<cudaStream_t>(stream), sp);
  if (e != cudaSuccess) return cuda_fail(e, "similarity kernel launch");
  return FB_OK;
}

fb_status fb_step(const fb_problem* problem, const fb_params* params, const fb_cache* cache, const fb_bf16* q,
                  const fb_bf16* k_in, const fb_bf16* v_in, const fb_bf16* k_out, const fb_bf16* v_out,
                  const int32_t* n_updated, const uint8_t* head_reuse_in, fb_bf16* a_full, float* l_full,
                  uint8_t* decision_out, void* workspace, size_t workspace_bytes, fb_stream_t stream) {
  const Range range("fb_step");
  FB_TRY(check_problem(problem));
  if (!params) return fail(FB_ERR_INVALID_ARG, "params is NULL");
  if (!cache) return fail(FB_ERR_INVALID_ARG, "cache is NULL");
  const unsigned flags = params->flags;
  if (flags & ~31u) return fail(FB_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags & ~31u);
  if ((flags & FB_FORCE_RECOMPUTE) && (flags & FB_FORCE_REUSE))
    return fail(FB_ERR_INVALID_ARG, "FB_FORCE_RECOMPUTE and FB_FORCE_REUSE are exclusive");
  if ((flags & FB_GATE_TAU) && (flags & FB_GATE_TAU_CUM))
    return fail(FB_ERR_INVALID_ARG, "FB_GATE_TAU and FB_GATE_TAU_CUM are exclusive");
  if ((flags & FB_GATE_TAU_CUM) && problem->num_seqs > 0 && (!n_updated || !cache->m_acc))
    return fail(FB_ERR_INVALID_ARG, "FB_GATE_TAU_CUM needs n_updated and cache->m_acc");
  const bool rows = problem->total_q > 0;
  const bool uses_gates = !(flags & (FB_FORCE_RECOMPUTE | FB_FORCE_REUSE)) && !head_reuse_in;
  const bool head_gate = uses_gates && (flags & FB_GATE_HEAD);
  if (uses_gates && (flags & FB_GATE_TAU) && !n_updated)
    return fail(FB_ERR_INVALID_ARG, "FB_GATE_TAU needs n_updated");
  if (head_gate && !cache->q_ref) return fail(FB_ERR_INVALID_ARG, "FB_GATE_HEAD needs cache->q_ref");
  if (head_gate && !(params->gamma == params->gamma)) return fail(FB_ERR_INVALID_ARG, "gamma is NaN");
  FB_TRY(check_ptr(q, "q", rows));
  FB_TRY(check_ptr(k_in, "k_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(v_in, "v_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(k_out, "k_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(v_out, "v_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(a_full, "a_full", rows));
  FB_TRY(check_ptr(cache->a_out, "cache->a_out", problem->total_kv_in > 0));
  if (problem->total_kv_in > 0 && !cache->l_out) return fail(FB_ERR_INVALID_ARG, "cache->l_out is NULL");
  if (problem->num_seqs > 0 && !cache->valid) return fail(FB_ERR_INVALID_ARG, "cache->valid is NULL");
  if (cache->q_ref) FB_TRY(check_ptr(cache->q_ref, "cache->q_ref", true));
  if (problem->num_seqs == 0) return FB_OK;
  const Plan pl = make_plan(problem, device_sms(), false, true);
  if (!workspace || workspace_bytes < pl.bytes)
    return fail(FB_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, pl.bytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  fb::Params prm;
  std::memset(&prm, 0, sizeof(prm));
  fill_problem(problem, pl, prm);
  fill_workspace(pl, workspace, prm);
  FB_TRY(kv_map(k_out, problem->total_kv_out, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_k_out));
  FB_TRY(kv_map(v_out, problem->total_kv_out, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_v_out));
  FB_TRY(kv_map(k_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_k_in));
  FB_TRY(kv_map(v_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, pl.bn, &prm.tm_v_in));

  if (head_gate) {  // with no active rows every score is 0 (a zero denominator), never a stale one
    float* cos_ws = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.off_cos);
    FB_TRY(fb_head_similarity(problem, q, cache->q_ref, cos_ws, stream));
  }
  const bool order_work = pl.tc2 && uses_gates && rows;  // decisions may differ per head
  prm.q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm.do_out = 1;
  prm.do_in = 1;
  prm.fused = 1;
  prm.update_state = 1;
  prm.flags = flags;
  prm.tau = params->tau;
  prm.gamma = params->gamma;
  prm.n_updated = n_updated;
  prm.head_reuse_in = head_reuse_in;
  prm.cache_a = cache->a_out;
  prm.cache_l = cache->l_out;
  prm.valid = cache->valid;
  prm.m_acc = cache->m_acc;
  prm.q_ref = reinterpret_cast<__nv_bfloat16*>(cache->q_ref);
  prm.a_full = reinterpret_cast<__nv_bfloat16*>(a_full);
  prm.l_full = l_full;
  prm.decision_out = decision_out;
  if (pl.reuse && problem->total_q > 0 && problem->total_kv_in > 0) {
    // block K/V with 64-row boxes and the Q box of a lean CTA
    FB_TRY(kv_map(k_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, fb::kBN, &prm.tm_k_lean));
    FB_TRY(kv_map(v_in, problem->total_kv_in, problem->num_heads_kv, problem->head_dim, fb::kBN, &prm.tm_v_lean));
    FB_TRY(q_map(q, problem->total_q, problem->num_heads_q, problem->head_dim, pl.g, pl.reuse_bt, &prm.tm_q_lean));
    prm.reuse_chunks = pl.reuse_chunks;
    prm.reuse_bt = pl.reuse_bt;
    prm.lean_early = pl.reuse_early ? 1 : 0;
    prm.lean = 1;
  }
  if (order_work) {
    int* order = reinterpret_cast<int*>(static_cast<char*>(workspace) + pl.off_order);
    if (pl.n_groups != pl.order_items)
      return fail(FB_ERR_INVALID_ARG, "internal: %d work items, order sized for %d", pl.n_groups, pl.order_items);
    int* order_arg = order;
    cudaError_t e = launch_pdl(fb::order_kernel, 1, fb::kOrderThreads, st, prm, order_arg);
    if (e != cudaSuccess) return cuda_fail(e, "order kernel launch");
    prm.order = order;
  }
  return launch_attn(pl, prm, st);
}

fb_status fb_cache_invalidate(const fb_problem* problem, const fb_cache* cache, fb_stream_t stream) {
  const Range range("fb_cache_invalidate");
  FB_TRY(check_problem(problem));
  if (!cache || (!cache->valid && problem->num_seqs > 0)) return fail(FB_ERR_INVALID_ARG, "cache->valid is NULL");
  const size_t n = static_cast<size_t>(problem->num_seqs) * problem->num_heads_q;
  if (!n) return FB_OK;
  cudaError_t e = cudaMemsetAsync(cache->valid, 0, n, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(valid)");
  return FB_OK;
}

fb_status fb_cache_copy_seq(const fb_problem* problem, const fb_cache* cache, int32_t src_seq, int32_t dst_seq,
                            fb_stream_t stream) {
  const Range range("fb_cache_copy_seq");
  FB_TRY(check_problem(problem));
  if (!cache) return fail(FB_ERR_INVALID_ARG, "cache is NULL");
  if (src_seq < 0 || src_seq >= problem->num_seqs || dst_seq < 0 || dst_seq >= problem->num_seqs)
    return fail(FB_ERR_INVALID_ARG, "sequence index out of range (src %d, dst %d, num_seqs %d)", src_seq, dst_seq,
                problem->num_seqs);
  if (src_seq == dst_seq) return FB_OK;
  if (!cache->valid) return fail(FB_ERR_INVALID_ARG, "cache->valid is NULL");
  FB_TRY(check_ptr(cache->a_out, "cache->a_out", problem->total_kv_in > 0));
  if (problem->total_kv_in > 0 && !cache->l_out) return fail(FB_ERR_INVALID_ARG, "cache->l_out is NULL");
  if (cache->q_ref) FB_TRY(check_ptr(cache->q_ref, "cache->q_ref", true));
  fb::CacheCopyParams cp{problem->num_heads_q, problem->head_dim, problem->num_seqs, problem->total_kv_in, src_seq,
                         dst_seq, problem->cu_seqlens_kv_in, cache->a_out, cache->l_out, cache->valid,
                         reinterpret_cast<__nv_bfloat16*>(cache->q_ref), cache->m_acc};
  const long items = static_cast<long>(std::max(problem->max_kv_in, 1)) * problem->num_heads_q * (problem->head_dim / 4);
  const int blocks = static_cast<int>(std::min<long>((items + 255) / 256, 148 * 8));
  cudaError_t e = launch_pdl(fb::cache_copy_kernel, std::max(blocks, 1), 256, reinterpret_cast<cudaStream_t>(stream), cp);
  if (e != cudaSuccess) return cuda_fail(e, "cache copy kernel launch");
  return FB_OK;
}

fb_status fb_cache_invalidate_seqs(const fb_problem* problem, const fb_cache* cache, const uint8_t* seq_mask,
                                   fb_stream_t stream) {
  const Range range("fb_cache_invalidate_seqs");
  FB_TRY(check_problem(problem));
  if (!cache || (!cache->valid && problem->num_seqs > 0)) return fail(FB_ERR_INVALID_ARG, "cache->valid is NULL");
  if (problem->num_seqs == 0) return FB_OK;
  fb::InvalidateParams ip{problem->num_heads_q, problem->num_seqs, seq_mask, cache->valid, cache->m_acc};
  const int total = problem->num_seqs * problem->num_heads_q;
  const int blocks = std::min((total + 255) / 256, 148);
  cudaError_t e = launch_pdl(fb::cache_invalidate_kernel, blocks, 256, reinterpret_cast<cudaStream_t>(stream), ip);
  if (e != cudaSuccess) return cuda_fail(e, "cache invalidate kernel launch");
  return FB_OK;
}

fb_status fb_sparse_layout(const fb_problem* problem, const int32_t* cu_sel, const int32_t* sel_idx,
                           int32_t total_sel, const fb_bf16* k_out, const fb_bf16* v_out, const fb_bf16* k_in,
                           const fb_bf16* v_in, fb_bf16* k_ext, fb_bf16* v_ext, uint32_t* kv_out_skip,
                           int32_t* cu_seqlens_kv_in_ext, fb_stream_t stream) {
  const Range range("fb_sparse_layout");
  FB_TRY(check_problem(problem));
  if (total_sel < 0 || total_sel > problem->total_kv_out)
    return fail(FB_ERR_INVALID_ARG, "total_sel %d outside [0, total_kv_out]", total_sel);
  if (problem->num_seqs == 0) return FB_OK;
  if (problem->num_seqs > 65535)  // one grid row per sequence
    return fail(FB_ERR_UNSUPPORTED, "fb_sparse_layout takes at most 65535 sequences per call");
  if (!cu_sel) return fail(FB_ERR_INVALID_ARG, "cu_sel is NULL");
  if (total_sel > 0 && !sel_idx) return fail(FB_ERR_INVALID_ARG, "sel_idx is NULL");
  const bool ext = problem->total_kv_in + total_sel > 0;
  FB_TRY(check_ptr(k_out, "k_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(v_out, "v_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(k_in, "k_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(v_in, "v_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(k_ext, "k_ext", ext));
  FB_TRY(check_ptr(v_ext, "v_ext", ext));
  if (problem->total_kv_out > 0 && !kv_out_skip) return fail(FB_ERR_INVALID_ARG, "kv_out_skip is NULL");
  if (kv_out_skip && (reinterpret_cast<uintptr_t>(kv_out_skip) & 3u))
    return fail(FB_ERR_INVALID_ARG, "kv_out_skip is not 4-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fb::SparseParams sp{problem->num_seqs, problem->num_heads_kv, problem->head_dim, problem->total_kv_out,
                      problem->total_kv_in, total_sel, problem->cu_seqlens_kv_out, problem->cu_seqlens_kv_in, cu_sel,
                      sel_idx, reinterpret_cast<const __nv_bfloat16*>(k_out),
                      reinterpret_cast<const __nv_bfloat16*>(v_out), reinterpret_cast<const __nv_bfloat16*>(k_in),
                      reinterpret_cast<const __nv_bfloat16*>(v_in), reinterpret_cast<__nv_bfloat16*>(k_ext),
                      reinterpret_cast<__nv_bfloat16*>(v_ext), kv_out_skip, cu_seqlens_kv_in_ext};
  // rows of J_in' per sequence: the block plus the selection (at most the prefix)
  const long per_seq = static_cast<long>(problem->max_kv_in + std::min(problem->max_kv_out, total_sel)) *
                       problem->num_heads_kv * problem->head_dim / 8;
  const int bx = static_cast<int>(std::max<long>(1, std::min<long>((per_seq + 255) / 256, 256)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bx, problem->num_seqs);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&sp};
  cudaError_t e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(&fb::sparse_layout_kernel), args);
  if (e != cudaSuccess) return cuda_fail(e, "sparse layout kernel launch");
  return FB_OK;
}

fb_status fb_prefix_append(const fb_problem* problem, const fb_bf16* k_out, const fb_bf16* v_out,
                           const fb_bf16* k_in, const fb_bf16* v_in, fb_bf16* k_dst, fb_bf16* v_dst,
                           int32_t* cu_seqlens_kv_out_dst, fb_stream_t stream) {
  const Range range("fb_prefix_append");
  FB_TRY(check_problem(problem));
  if (problem->num_seqs == 0) return FB_OK;
  if (problem->num_seqs > 65535)  // one grid row per sequence
    return fail(FB_ERR_UNSUPPORTED, "fb_prefix_append takes at most 65535 sequences per call");
  const bool in_place = k_dst == k_out && problem->total_kv_out > 0;
  if (in_place != (v_dst == v_out && problem->total_kv_out > 0))
    return fail(FB_ERR_INVALID_ARG, "K and V must both be appended in place or both into new buffers");
  if (in_place && problem->num_seqs != 1)
    return fail(FB_ERR_UNSUPPORTED, "in-place append takes one sequence (later sequences would have to move)");
  const long grown = static_cast<long>(problem->total_kv_out) + problem->total_kv_in;
  if (grown >= (1L << 31)) return fail(FB_ERR_UNSUPPORTED, "grown prefix of %ld tokens", grown);
  FB_TRY(check_ptr(k_out, "k_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(v_out, "v_out", problem->total_kv_out > 0));
  FB_TRY(check_ptr(k_in, "k_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(v_in, "v_in", problem->total_kv_in > 0));
  FB_TRY(check_ptr(k_dst, "k_dst", grown > 0));
  FB_TRY(check_ptr(v_dst, "v_dst", grown > 0));
  fb::AppendParams ap{problem->num_seqs, problem->num_heads_kv, problem->head_dim, problem->total_kv_out,
                      problem->total_kv_in, in_place ? 0 : 1, problem->cu_seqlens_kv_out, problem->cu_seqlens_kv_in,
                      reinterpret_cast<const __nv_bfloat16*>(k_out), reinterpret_cast<const __nv_bfloat16*>(v_out),
                      reinterpret_cast<const __nv_bfloat16*>(k_in), reinterpret_cast<const __nv_bfloat16*>(v_in),
                      reinterpret_cast<__nv_bfloat16*>(k_dst), reinterpret_cast<__nv_bfloat16*>(v_dst),
                      cu_seqlens_kv_out_dst};
  const long per_seq = static_cast<long>((in_place ? 0 : problem->max_kv_out) + problem->max_kv_in) *
                       problem->num_heads_kv * problem->head_dim / 8;
  const int bx = static_cast<int>(std::max<long>(1, std::min<long>((per_seq + 255) / 256, 1184)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bx, problem->num_seqs);
  cfg.blockDim = dim3(256);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&ap};
  cudaError_t e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(&fb::prefix_append_kernel), args);
  if (e != cudaSuccess) return cuda_fail(e, "prefix append kernel launch");
  return FB_OK;
}

fb_status fb_selftest_wait_timeout(fb_stream_t stream) {
  const Range range("fb_selftest_wait_timeout");
  fb::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test kernel launch");
  return FB_OK;
}

fb_status fb_release_cache(void) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  g_maps.clear();
  return FB_OK;
}

fb_status fb_device_status(int32_t* code, fb_stream_t stream) {
  const Range range("fb_device_status");
  if (!code) return fail(FB_ERR_INVALID_ARG, "code is NULL");
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, fb::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  const int zero = 0;
  e = cudaMemcpyToSymbol(fb::g_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  *code = v;
  return FB_OK;
}

}  // extern "C"
