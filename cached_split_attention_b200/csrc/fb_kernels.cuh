// FlashBlock denoise-step attention kernels (sm_100a).
//
// `attn_kernel` serves the out-of-block pass (J_out, the cached prefix), the
// in-block pass (J_in, the block's own tokens, bidirectional) and the fused step.
//
// Work decomposition.  A group is (sequence b, kv-head hk, row tile t); a row is a
// (query token, q-head of the kv-head's group) pair, so one kv-head's K/V is
// streamed once for all of its q-heads (grouped-query attention).  Each group is
// handled by S CTAs that form one thread-block cluster.  The group's prefix key
// chunks (64 keys each) are dealt out over the S CTAs; the block's chunks, when the
// block pass runs, go to the last CTA, whose prefix share is shortened to match.
// Every CTA computes partials (A, L) with A normalised and L = ln Z (FlashBlock,
// "Mecanismo Central") and keeps them in shared memory: the block partial in a
// region of its own (the block segment runs first), the prefix partial in the
// drained stage ring.
//
// Merge.  The log-space composition
//     A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m})
// is associative, so combining the S prefix partials and adding the block partial
// are the same operation.  With S > 1 and a head that recomputes, the cluster
// synchronises and each CTA merges a slice of the rows, reading the partials of
// the other CTAs through distributed shared memory; otherwise the CTA that holds
// all partials merges every row.  The merge writes the cache for heads that
// recompute, reads it for heads that reuse, and writes A_full / L_full.  No CTA
// waits on another CTA outside the cluster barriers; the last CTA of the grid (an
// atomic counter) marks recomputed heads valid and writes the decisions.
//
// Inside a CTA: thread 0 streams K/V chunks with TMA (128-byte swizzle,
// evict-first L2 policy) through a ring of mbarrier-guarded stages.  Warp
// (wm, wn) owns 16 rows and a 1/WN share of the keys of every stage and runs
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) with an online softmax in base 2;
// each warp hands off its own sub-partial and the merge combines all of them.
#pragma once

#include <limits>

#include "fb_device.cuh"

namespace fb {

constexpr unsigned kGateTau = 1u, kGateHead = 2u, kForceRecompute = 4u, kForceReuse = 8u, kGateTauCum = 16u;
constexpr int kBN = 64;        // keys per pipeline stage
constexpr int kMaxGroup = 32;  // q-heads per kv-head
constexpr int kMaxSplits = 8;  // CTAs per cluster (portable limit)
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -std::numeric_limits<float>::infinity();

__device__ int g_status;  // first error recorded by any kernel (0 = none)

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// Bits [t0, t0 + 64) of a prefix-token bitmask (bit t % 32 of word t / 32) as one
// 64-bit word, bit k = token t0 + k; words past the end (total_out tokens) read 0.
__device__ __forceinline__ uint64_t skip_bits64(const uint32_t* bits, int total_out, int t0) {
  const int nwords = (total_out + 31) >> 5;
  const int w = t0 >> 5;
  const int sh = t0 & 31;
  auto word = [&](int i) -> uint64_t { return i < nwords ? static_cast<uint64_t>(__ldg(bits + i)) : 0ull; };
  const uint64_t lo = word(w) | (word(w + 1) << 32);
  return sh ? (lo >> sh) | (word(w + 2) << (64 - sh)) : lo;
}

struct alignas(64) Params {
  CUtensorMap tm_k_out, tm_v_out, tm_k_in, tm_v_in;
  // problem
  int num_seqs, hq, hkv, g;
  float scale_log2;  // softmax scale * log2(e)
  const int* cu_q;
  const int* q_rows;
  const int* cu_out;
  const int* cu_in;
  const __nv_bfloat16* q;
  int total_q, total_out, total_in;  // host totals: every index is checked against them
  // plan
  int tiles, splits;
  // mode
  int do_out, do_in, fused, update_state;
  // gates
  unsigned flags;
  int tau;
  float gamma;
  const int* n_updated;
  const uint8_t* head_reuse_in;
  const uint8_t* head_mask;
  const float* cos;
  // cache and outputs
  float* cache_a;
  float* cache_l;
  uint8_t* valid;
  int* m_acc;  // cumulative updated-token count per (b, h) (kGateTauCum)
  __nv_bfloat16* q_ref;
  __nv_bfloat16* a_full;
  float* l_full;
  uint8_t* decision_out;
  float* a_in;
  float* l_in;
  // workspace
  int* grid_ctr;     // completion counter of the cache-state epilogue (zero between calls)
  const int* order;  // work order of the two-tile kernel (NULL: CTA i takes item i)
  const uint32_t* out_skip;  // prefix tokens left out of J_out (bitmask; NULL: none)
  // lean reuse path (fb_reuse.cuh)
  CUtensorMap tm_k_lean, tm_v_lean;  // block K/V with 64-row boxes (the warp-MMA stage layout)
  CUtensorMap tm_q_lean;             // Q as {d, hq, tokens}, box {64, g, reuse_bt}
  int reuse_chunks;  // 64-key chunks of the longest block
  int reuse_bt;      // tokens of a lean CTA's Q box
  int lean_early;    // 1: lean loads go out before the reuse decision (one-wave grids)
  int lean;          // 1: groups whose heads all reuse take the lean path
};

// Bring the kernel's tensor-map descriptors on chip while the previous kernel of
// the stream finishes (they live in this launch's parameters, which no earlier
// kernel writes, so this may run before pdl_wait).
__device__ __forceinline__ void prefetch_maps(const Params& p) {
  if (threadIdx.x != 0) return;
  if (p.total_out > 0) {
    prefetch_tensormap(&p.tm_k_out);
    prefetch_tensormap(&p.tm_v_out);
  }
  if (p.total_in > 0) {
    prefetch_tensormap(&p.tm_k_in);
    prefetch_tensormap(&p.tm_v_in);
    if (p.lean) {
      prefetch_tensormap(&p.tm_k_lean);
      prefetch_tensormap(&p.tm_v_lean);
      prefetch_tensormap(&p.tm_q_lean);
    }
  }
}

// Reuse decision of (b, h) (true: recompute); see fb_step in flashblock.h.
// Inputs of the decision of (b, h), loaded in one go (every load goes out before
// any is tested: one memory round trip instead of a dependent chain) and tested by
// decide(), so that a caller can do other work while they are in flight.
struct DecisionIn {
  int b, idx;
  int mask, valid, reuse_in, n_upd, m_acc;
  float cs;
};
__device__ __forceinline__ DecisionIn decision_load(const Params& p, int b, int h) {
  DecisionIn d;
  d.b = b;
  d.idx = b * p.hq + h;
  d.mask = d.valid = d.reuse_in = 1;
  d.n_upd = d.m_acc = 0;
  d.cs = 0.f;
  if (!p.update_state) {
    if (p.head_mask) d.mask = p.head_mask[d.idx];
    return d;
  }
  if (p.flags & kForceRecompute) return d;
  const bool tau = (p.flags & (kGateTau | kGateTauCum)) && p.n_updated;
  d.valid = p.valid[d.idx];
  d.reuse_in = p.head_reuse_in ? p.head_reuse_in[d.idx] : 1;
  d.n_upd = tau ? p.n_updated[b] : 0;
  d.m_acc = ((p.flags & kGateTauCum) && p.m_acc) ? p.m_acc[d.idx] : 0;
  d.cs = (p.flags & kGateHead) ? p.cos[d.idx] : 0.f;
  return d;
}
__device__ __forceinline__ bool decide(const Params& p, const DecisionIn& d) {
  if (!p.update_state) return d.mask != 0;
  if (p.flags & kForceRecompute) return true;
  if (!d.valid) return true;
  if (p.flags & kForceReuse) return false;
  if (p.head_reuse_in) return d.reuse_in == 0;
  bool reuse = true;
  if (p.flags & kGateTau) reuse = reuse && (d.n_upd < p.tau);
  if (p.flags & kGateTauCum) reuse = reuse && (d.m_acc + d.n_upd < p.tau);
  if (p.flags & kGateHead) reuse = reuse && (d.cs > p.gamma);
  return !reuse;
}
__device__ __forceinline__ bool head_recompute(const Params& p, int b, int h) {
  return decide(p, decision_load(p, b, h));
}

// The state vote's loads, issued here and tested in state_vote (so that the
// decision's loads go out beside them): at most 8 `valid` entries per thread.
struct VoteLoads {
  uint8_t e[8];  // the entries (1 where there is none)
  bool all;      // every call updates state
};
__device__ __forceinline__ VoteLoads state_vote_load(const Params& p, int tid, int nthreads) {
  VoteLoads v;
  const int total = p.num_seqs * p.hq;
  v.all = p.update_state && ((p.flags & kGateTauCum) || total > 8 * nthreads);
  const bool load = p.update_state && !v.all;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int i = tid + k * nthreads;
    v.e[k] = (load && i < total) ? p.valid[i] : uint8_t(1);
  }
  return v;
}

// Whether this call's last CTA has cache state to update: a head whose entry is
// still empty (it becomes valid), or the cumulative count (kept on every call).
// Every thread of the CTA calls it; the result is CTA-uniform through the vote.
__device__ __forceinline__ bool state_vote(const VoteLoads& v) {
  int need = v.all;
#pragma unroll
  for (int k = 0; k < 8; ++k) need |= v.e[k] == 0;
  return __syncthreads_or(need) != 0;
}

// Cache-state epilogue: every CTA has read `valid` and `m_acc` (its decisions)
// before it arrives on the completion counter; the last one to arrive marks the
// heads that recomputed valid and advances the cumulative counts (0 after a
// recompute, + n_updated after a reuse).  No CTA waits; the last one also resets
// the counter for the next call.
__device__ __forceinline__ void state_epilogue(const Params& p, int tid, int nthreads, int* s_flag) {
  __syncthreads();
  if (tid == 0) *s_flag = (atomicAdd(p.grid_ctr, 1) == static_cast<int>(gridDim.x) - 1) ? 1 : 0;
  __syncthreads();
  if (*s_flag) {
    __threadfence();
    const int total = p.num_seqs * p.hq;
    for (int idx = tid; idx < total; idx += nthreads) {
      const int b = idx / p.hq;
      const bool rec = head_recompute(p, b, idx % p.hq);
      if (rec) p.valid[idx] = 1;
      if (p.flags & kGateTauCum) p.m_acc[idx] = rec ? 0 : p.m_acc[idx] + p.n_updated[b];
    }
    if (tid == 0) *p.grid_ctr = 0;
  }
}

// Prefix chunks [a, b) of CTA s of S.  The last CTA also runs the `in_chunks`
// block chunks, so it takes fewer prefix chunks; the rest are spread evenly.
__device__ __forceinline__ void prefix_range(int s, int S, int out_chunks, int in_chunks, int& a, int& b) {
  if (S == 1) {
    a = 0;
    b = out_chunks;
    return;
  }
  // the block segment costs its chunks plus about two chunks of hand-off
  const int in_cost = in_chunks > 0 ? in_chunks + 2 : 0;
  const int per = (out_chunks + in_cost + S - 1) / S;
  const int last = min(out_chunks, max(0, per - in_cost));
  const int rest = out_chunks - last;
  if (s == S - 1) {
    a = rest;
    b = out_chunks;
    return;
  }
  const int q = rest / (S - 1), r = rest % (S - 1);
  a = s * q + min(s, r);
  b = a + q + (s < r ? 1 : 0);
}

// Log-space sum of N normalised partials with base-2 log-normalisers l2[k]
// (empty partials: -inf):  out = sum_k 2^{l2[k]-m} a[k] / sum_k 2^{l2[k]-m},
// returning m + log2 sum_k 2^{l2[k]-m} (m = max_k l2[k]); (0, -inf) when every
// partial is empty.  Hardware ex2 / lg2 / rcp approximations (relative error
// about 2^-22), well below the bf16 output resolution.
template <int N>
__device__ __forceinline__ float lse2_combine(const float (&l2)[N], const float4 (&a)[N], float4& out) {
  float mx = kNegInf;
#pragma unroll
  for (int k = 0; k < N; ++k) mx = fmaxf(mx, l2[k]);
  out = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx == kNegInf) return kNegInf;
  float den = 0.f;
#pragma unroll
  for (int k = 0; k < N; ++k) {
    if (l2[k] == kNegInf) continue;  // empty partial (its A may be unset)
    const float w = ex2(l2[k] - mx);
    den += w;
    out.x = fmaf(w, a[k].x, out.x);
    out.y = fmaf(w, a[k].y, out.y);
    out.z = fmaf(w, a[k].z, out.z);
    out.w = fmaf(w, a[k].w, out.w);
  }
  const float inv = rcp_approx(den);
  out.x *= inv;
  out.y *= inv;
  out.z *= inv;
  out.w *= inv;
  return mx + lg2_approx(den);
}

// Weights of the log-space sum of N partials with base-2 log-normalisers l2[k]:
// w[k] = 2^{l2[k]-m} / sum_j 2^{l2[j]-m}; returns m + log2 sum_j 2^{l2[j]-m}
// (m = max l2), or -inf with all weights 0 when every partial is empty.
template <int N>
__device__ __forceinline__ float log2_weights(const float (&l2)[N], float* w) {
  float mx = kNegInf;
#pragma unroll
  for (int k = 0; k < N; ++k) mx = fmaxf(mx, l2[k]);
  if (mx == kNegInf) {
#pragma unroll
    for (int k = 0; k < N; ++k) w[k] = 0.f;
    return kNegInf;
  }
  float e[N];
  float den = 0.f;
#pragma unroll
  for (int k = 0; k < N; ++k) {
    e[k] = l2[k] == kNegInf ? 0.f : ex2(l2[k] - mx);
    den += e[k];
  }
  const float inv = rcp_approx(den);
#pragma unroll
  for (int k = 0; k < N; ++k) w[k] = e[k] * inv;
  return mx + lg2_approx(den);
}

__device__ __forceinline__ void fma4(float4& acc, float w, const float4& v) {
  acc.x = fmaf(w, v.x, acc.x);
  acc.y = fmaf(w, v.y, acc.y);
  acc.z = fmaf(w, v.z, acc.z);
  acc.w = fmaf(w, v.w, acc.w);
}

// Store the folded (natural-log) normaliser of row r of a partial.
__device__ __forceinline__ void part_l_fold(float* part, int off_l, int r, float lse2) {
  part[off_l + r] = lse2 == kNegInf ? kNegInf : lse2 * kLn2;
}

template <int D, int WM, int WN, int STAGES>
struct Cfg {
  static constexpr int kRows = 16 * WM;
  static constexpr int kWarps = WM * WN;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kKW = kBN / WN;            // keys of a stage per warp
  static constexpr int kTileBytes = kBN * D * 2;  // K (or V) tile of one stage
  static constexpr int kHalfBytes = kBN * 128;    // one 64-column swizzle span
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStageArea = STAGES * kStageBytes;
  static constexpr int kQStride = D + 8;  // padded Q row, elements
  static constexpr int kQBytes = kRows * kQStride * 2;
  static constexpr int kPStride = D + 4;  // padded partial row, floats
  // A partial of the tile is WN sub-partials, one per key share:
  // A [WN][kRows][kPStride] floats, then L [WN][kRows] floats.
  static constexpr int kPartL = WN * kRows * kPStride;  // offset of L, floats
  static constexpr int kPartBytes = (kPartL + WN * kRows) * 4;
  static constexpr int kOffQ = kStageArea;
  static constexpr int kOffIn = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffIn + kPartBytes;
  static constexpr int kOffPos = kOffBar + 2 * STAGES * 8;
  // Cached A_out / L_out rows of heads that reuse, copied in while the attention
  // runs (tiles of up to 32 rows; larger tiles read them from L2 at the merge).
  static constexpr bool kStageCache = kRows <= 32;
  static constexpr int kOffCache = (kOffPos + kRows * 4 + 15) / 16 * 16;
  static constexpr int kCacheBytes = kStageCache ? kRows * kPStride * 4 + kRows * 4 : 0;
  static constexpr int kSmem = 1024 + kOffCache + kCacheBytes;
  static_assert(kKW % 16 == 0, "keys per warp must be a multiple of 16");
  static_assert(kPartBytes <= kStageArea, "the prefix partial must fit in the stage ring");
  static_assert(kOffIn % 16 == 0 && kOffBar % 8 == 0, "aligned regions");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(32 % (D / 4) == 0 && kThreads % 32 == 0, "a row's float4 items share one warp");
  static_assert(kRows * (kMaxSplits + WN + 6) * 4 <= kQBytes, "per-row merge weights fit in the Q tile");
};

// Byte offset of (key row kr, column dd) inside a stage tile written by TMA with
// 128-byte swizzle: 16-byte chunk c of a 128-byte row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int kr, int dd) {
  return static_cast<uint32_t>((dd >> 6) * (kBN * 128) + kr * 128 + ((((dd & 63) >> 3) ^ (kr & 7)) << 4));
}

// Running softmax state of one warp: 16 rows; a thread holds rows lane/4 and lane/4+8.
template <int D>
struct Acc {
  float o[D / 8][4];
  float m[2];
  float l[2];  // per-thread partial sums; quad-reduced when finished
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    m[0] = m[1] = kNegInf;
    l[0] = l[1] = 0.f;
  }
};

// KW keys of one stage: S = Q K^T, online softmax, O += P V.  `kr0` is the first
// key row of the warp inside the stage tile.
template <int D, int KW>
__device__ __forceinline__ void consume_keys(Acc<D>& acc, const uint32_t (&qf)[D / 16][4], uint32_t kb, uint32_t vb,
                                             int kr0, int key0, int k_end, float scale_log2, int lane,
                                             uint64_t skip = 0ull) {
  float s[KW / 8][4];
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int nb = 0; nb < KW / 16; ++nb) {
      const int mi = lane >> 3;
      const int kr = kr0 + nb * 16 + (mi >> 1) * 8 + (lane & 7);
      const int dd = kk * 16 + (mi & 1) * 8;
      uint32_t r[4];
      ldsm_x4(r, kb + swz(kr, dd));
      mma_bf16_16816(s[2 * nb], qf[kk], r[0], r[1]);
      mma_bf16_16816(s[2 * nb + 1], qf[kk], r[2], r[3]);
    }
  }
  // keys past the segment's end, and keys the skip mask leaves out (bit k = key key0 + k)
  const bool need_mask = key0 + KW > k_end || skip != 0ull;
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = s[n][e] * scale_log2;
      const int rel = n * 8 + 2 * (lane & 3) + (e & 1);
      if (need_mask && (key0 + rel >= k_end || ((skip >> rel) & 1ull))) v = kNegInf;
      s[n][e] = v;
    }
  }
  float mx[2] = {acc.m[0], acc.m[1]};
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
    mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
    mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
  }
  float msafe[2], alpha[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    mx[i] = quad_max(mx[i]);
    msafe[i] = mx[i] == kNegInf ? 0.f : mx[i];
    alpha[i] = ex2(acc.m[i] - msafe[i]);
  }
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
    s[n][0] = ex2(s[n][0] - msafe[0]);
    s[n][1] = ex2(s[n][1] - msafe[0]);
    s[n][2] = ex2(s[n][2] - msafe[1]);
    s[n][3] = ex2(s[n][3] - msafe[1]);
    rs[0] += s[n][0] + s[n][1];
    rs[1] += s[n][2] + s[n][3];
  }
  // O only needs rescaling when some row's running max moved (exact either way).
  if (__any_sync(0xffffffffu, mx[0] != acc.m[0] || mx[1] != acc.m[1])) {
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc.o[n][0] *= alpha[0];
      acc.o[n][1] *= alpha[0];
      acc.o[n][2] *= alpha[1];
      acc.o[n][3] *= alpha[1];
    }
    acc.l[0] *= alpha[0];
    acc.l[1] *= alpha[1];
  }
  acc.m[0] = mx[0];
  acc.m[1] = mx[1];
  acc.l[0] += rs[0];
  acc.l[1] += rs[1];
#pragma unroll
  for (int kb2 = 0; kb2 < KW / 16; ++kb2) {
    uint32_t a[4];
    a[0] = pack_bf16x2(s[2 * kb2][0], s[2 * kb2][1]);
    a[1] = pack_bf16x2(s[2 * kb2][2], s[2 * kb2][3]);
    a[2] = pack_bf16x2(s[2 * kb2 + 1][0], s[2 * kb2 + 1][1]);
    a[3] = pack_bf16x2(s[2 * kb2 + 1][2], s[2 * kb2 + 1][3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      const int mi = lane >> 3;
      const int kr = kr0 + kb2 * 16 + (mi & 1) * 8 + (lane & 7);
      const int dd = np * 16 + (mi >> 1) * 8;
      uint32_t r[4];
      ldsm_x4_t(r, vb + swz(kr, dd));
      mma_bf16_16816(acc.o[2 * np], a, r[0], r[1]);
      mma_bf16_16816(acc.o[2 * np + 1], a, r[2], r[3]);
    }
  }
}

}  // namespace fb

#include "fb_reuse.cuh"  // the lean reuse path (uses the helpers above)

namespace fb {

template <int D, int WM, int WN, int STAGES>
__global__ void __launch_bounds__(Cfg<D, WM, WN, STAGES>::kThreads, 1) attn_kernel(const __grid_constant__ Params p) {
  prefetch_maps(p);
  using C = Cfg<D, WM, WN, STAGES>;
  constexpr int TR = C::kRows;
  constexpr int KW = C::kKW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  __nv_bfloat16* q_s = reinterpret_cast<__nv_bfloat16*>(smem + C::kOffQ);
  float* in_part = reinterpret_cast<float*>(smem + C::kOffIn);  // block partial
  float* out_part = reinterpret_cast<float*>(stages);            // prefix partial, after the ring drains
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + STAGES;
  int* s_pos = reinterpret_cast<int*>(smem + C::kOffPos);  // block position of each tile row (-1: none)
  float* cache_s = reinterpret_cast<float*>(smem + C::kOffCache);  // staged cache rows (kStageCache)
  __shared__ uint8_t s_rec[kMaxGroup];
  __shared__ int s_flag;
  __shared__ __align__(8) uint64_t s_lean_bar[2];  // lean path: inputs, cached rows

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int wm = warp % WM;
  const int wn = warp / WM;
  const int S = p.splits;
  const int split = blockIdx.x % S;  // == rank in the cluster
  const int gidx = blockIdx.x / S;
  const int t = gidx % p.tiles;
  const int bh = gidx / p.tiles;
  const int hk = bh % p.hkv;
  const int b = bh / p.hkv;
  const int g = p.g;

  // ------------------------------------------------------------ group metadata
  // The index arrays are read before the wait for the previous kernel of the
  // stream (no kernel that lets this one start early writes them; flashblock.h),
  // so these loads overlap its tail; the cache state is read after the wait.
  const int q0 = p.cu_q[b];
  const int n_q = p.cu_q[b + 1] - q0;
  const int out0 = p.cu_out[b];
  const int n_out = p.cu_out[b + 1] - out0;
  const int in0 = p.cu_in[b];
  const int n_in = p.cu_in[b + 1] - in0;
  const bool ranges_ok = q0 >= 0 && n_q >= 0 && q0 + n_q <= p.total_q && out0 >= 0 && n_out >= 0 &&
                         out0 + n_out <= p.total_out && in0 >= 0 && n_in >= 0 && in0 + n_in <= p.total_in &&
                         n_q <= n_in;
  if (!ranges_ok && tid == 0 && t == 0 && split == 0) record_status(kDevBadIndex);
  const int rows = ranges_ok ? n_q * g : 0;
  const int row0 = t * TR;
  const int nrows = max(0, min(TR, rows - row0));
  // Lean reuse path (fb_reuse.cuh): this CTA's rows of the group; in a one-wave
  // grid their Q and the block K/V are loaded while the previous kernel finishes.
  LeanRows lr{};
  const LeanSmem<D> ls(smem, p.reuse_chunks, g, p.reuse_bt);
  int lean_p = -1;  // block position of this thread's box token
  if (p.lean && nrows > 0 && n_in <= p.reuse_chunks * kBN) {
    int r0, nr;
    lean_rows(nrows, split, S, r0, nr);
    if (nr > 0) lr = lean_place(g, row0 + r0, nr);
  }
  const bool lean_early = lr.nr > 0 && p.lean_early;
  if (lr.nr > 0) lean_p = lean_pos(p, q0, lr, tid);
  if (lean_early) lean_issue<D>(p, ls, s_lean_bar, hk, q0, in0, n_in, lr, tid);
  pdl_wait();
  pdl_trigger();
  // The decision's loads, the state vote's and the early cache rows go out
  // together (the cache rows from warps 1.., after warp 0's decision loads).
  const VoteLoads vote = state_vote_load(p, tid, C::kThreads);
  DecisionIn din;
  if (tid < g) din = decision_load(p, b, hk * g + tid);
  if (lean_early) lean_fetch<D>(p, ls, s_lean_bar, hk, in0, n_in, lr, lean_p, tid);
  if (tid < g) s_rec[tid] = decide(p, din) ? 1 : 0;
  const bool need_state = state_vote(vote);
  bool any_rec = false;
  for (int j = 0; j < g; ++j) any_rec |= (s_rec[j] != 0);

  // ------------------------------------------------------------ chunk schedule
  const bool do_out = p.do_out && any_rec;
  const int out_chunks = do_out ? (n_out + kBN - 1) / kBN : 0;
  const int in_chunks = p.do_in ? (n_in + kBN - 1) / kBN : 0;
  int pa, pb;  // my prefix chunks
  prefix_range(split, S, out_chunks, in_chunks, pa, pb);
  const bool has_in = p.do_in && split == S - 1;
  const bool has_out = do_out && (pb > pa || (out_chunks == 0 && split == 0));
  const bool cluster_mode = S > 1 && do_out;  // uniform over the cluster
  const bool active = nrows > 0;               // uniform over the cluster
  // The block segment (if any) runs first into a region of its own; the prefix
  // segment runs last, so its partial can reuse the drained ring.
  const int nA = has_in ? in_chunks : 0;
  const int nB = has_out ? pb - pa : 0;
  const int n_local = nA + nB;
  // Merging: all CTAs of a cluster share the rows; otherwise the CTA that holds
  // every partial merges all of them.
  const bool merger = cluster_mode || has_in || (S == 1 && has_out);

  // decisions of this group's heads (written once per (b, kv-head))
  if (p.decision_out && t == 0 && split == S - 1 && tid < g) p.decision_out[b * p.hq + hk * g + tid] = s_rec[tid];
  // A group whose heads all reuse takes the lean reuse path (its CTAs share the rows).
  const bool lean = p.lean && !any_rec && active;
  if (!lean && lean_early) lean_drain(s_lean_bar, tid);
  if (lean) {
    if (n_in > p.reuse_chunks * kBN) {
      if (tid == 0) record_status(kDevBadIndex);
    } else if (lr.nr > 0) {
      if (!lean_early) {
        lean_issue<D>(p, ls, s_lean_bar, hk, q0, in0, n_in, lr, tid);
        lean_fetch<D>(p, ls, s_lean_bar, hk, in0, n_in, lr, lean_p, tid);
      }
      lean_finish<D>(p, ls, s_lean_bar, lr, q0, hk, n_in, tid, C::kThreads);
    }
  } else if (active && (has_in || has_out || cluster_mode)) {
    // -------------------------------------------------------- Q rows first
    // (before the K/V flood, so their loads are not queued behind it)
    constexpr int kQVec = TR * (D / 8);
    constexpr int kQPer = (kQVec + C::kThreads - 1) / C::kThreads;
    uint4 qv[kQPer];
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * C::kThreads;
      const int r = v / (D / 8);
      const int c = v % (D / 8);
      qv[k] = make_uint4(0u, 0u, 0u, 0u);
      if (v < kQVec && r < nrows) {
        const int rho = row0 + r;
        qv[k] = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(q0 + rho / g) * p.hq + hk * g + rho % g) * D +
                                                c * 8);
      }
    }
    // block positions of the tile rows (also before the flood)
    constexpr int kPosPer = (TR + C::kThreads - 1) / C::kThreads;
    int posv[kPosPer];
#pragma unroll
    for (int k = 0; k < kPosPer; ++k) {
      const int r = tid + k * C::kThreads;
      posv[k] = -1;
      if (r < nrows) {
        const int it = (row0 + r) / g;
        posv[k] = p.q_rows ? p.q_rows[q0 + it] : it;
      }
    }
    // -------------------------------------------------------- TMA ring
    if (tid == 0) {
      for (int s = 0; s < STAGES; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], C::kWarps);
      }
      fence_barrier_init();
    }
    uint64_t pol = 0;
    auto issue = [&](int c) {
      const bool seg_in = c < nA;
      const int cc = seg_in ? c : c - nA;
      const CUtensorMap* tk = seg_in ? &p.tm_k_in : &p.tm_k_out;
      const CUtensorMap* tv = seg_in ? &p.tm_v_in : &p.tm_v_out;
      const int y = seg_in ? in0 + cc * kBN : out0 + (pa + cc) * kBN;
      const int st = c % STAGES;
      mbar_arrive_expect_tx(&full[st], C::kStageBytes);
      uint8_t* kd = stages + st * C::kStageBytes;
      uint8_t* vd = kd + C::kTileBytes;
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_2d(kd + hh * C::kHalfBytes, tk, &full[st], hk * D + hh * 64, y, pol);
        tma_load_2d(vd + hh * C::kHalfBytes, tv, &full[st], hk * D + hh * 64, y, pol);
      }
    };
    if (tid == 0 && n_local > 0) {
      pol = l2_policy_evict_first();
      for (int c = 0; c < min(STAGES, n_local); ++c) issue(c);
    }
    // cached rows this CTA merges with go to L2 while the attention runs
#pragma unroll
    for (int k = 0; k < kPosPer; ++k) {
      const int r = tid + k * C::kThreads;
      if (r >= TR) continue;
      int pos = posv[k];
      if (r < nrows) {
        const int rho = row0 + r;
        if (pos < 0 || pos >= n_in) {
          record_status(kDevBadIndex);
          pos = -1;
        } else if (merger && p.fused && !(do_out && s_rec[rho % g])) {
          const size_t ce = static_cast<size_t>(in0 + pos) * p.hq + hk * g + rho % g;
          if constexpr (C::kStageCache) {
            for (int c = 0; c < D / 4; ++c)
              cp_async_16(cache_s + r * C::kPStride + c * 4, p.cache_a + ce * D + c * 4);
            cp_async_4(cache_s + TR * C::kPStride + r, p.cache_l + ce);
          } else {
            prefetch_l2(p.cache_a + ce * D, D * 4);
            prefetch_l2_line(p.cache_l + ce);
          }
        }
      }
      s_pos[r] = pos;
    }
    cp_async_commit();
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * C::kThreads;
      if (v < kQVec) *reinterpret_cast<uint4*>(q_s + (v / (D / 8)) * C::kQStride + (v % (D / 8)) * 8) = qv[k];
    }
    __syncthreads();
    // q_ref follows the queries of heads that recompute (fb_step, block owner)
    if (has_in && p.fused && p.q_ref != nullptr && any_rec) {
      for (int v = tid; v < nrows * (D / 8); v += C::kThreads) {
        const int r = v / (D / 8);
        const int c = v % (D / 8);
        const int j = (row0 + r) % g;
        if (!s_rec[j] || s_pos[r] < 0) continue;
        const size_t e = (static_cast<size_t>(in0 + s_pos[r]) * p.hq + hk * g + j) * D + c * 8;
        *reinterpret_cast<uint4*>(p.q_ref + e) = *reinterpret_cast<const uint4*>(q_s + r * C::kQStride + c * 8);
      }
    }
    const bool rows_active = 16 * wm < nrows;
    uint32_t qf[D / 16][4];
    if (rows_active) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(qf[kk], smem_u32(q_s + (16 * wm + (lane & 15)) * C::kQStride + kk * 16 + (lane >> 4) * 8));
    }

    Acc<D> acc;
    acc.reset();
    bool ok = true;
    int issued = min(STAGES, n_local);

    // skip-mask bits of the warp's keys of a prefix chunk (loaded one chunk ahead)
    auto skip_of = [&](int c) -> uint64_t {
      if (!p.out_skip || c < nA || c >= n_local) return 0ull;
      uint64_t w = skip_bits64(p.out_skip, p.total_out, out0 + (pa + c - nA) * kBN + wn * KW);
      if constexpr (KW < 64) w &= (1ull << (KW % 64)) - 1ull;
      return w;
    };
    // One segment of chunks [c0, c1) of the local sequence.
    auto run = [&](int c0, int c1) {
      uint64_t skip_next = skip_of(c0);
      for (int c = c0; c < c1 && ok; ++c) {
        const uint64_t skip = skip_next;
        skip_next = skip_of(c + 1);
        const int st = c % STAGES;
        // every lane waits; the warp leaves together if the wait ran out
        if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (c / STAGES) & 1))) {
          record_status(kDevTimeout);
          ok = false;
          break;
        }
        if (rows_active) {
          const bool seg_in = c < nA;
          const int key0 = (seg_in ? c * kBN : (pa + c - nA) * kBN) + wn * KW;
          const uint32_t kb = smem_u32(stages + st * C::kStageBytes);
          consume_keys<D, KW>(acc, qf, kb, kb + C::kTileBytes, wn * KW, key0, seg_in ? n_in : n_out, p.scale_log2,
                              lane, skip);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (warp == 0 && c + STAGES < n_local) {
          bool refill_ok = true;
          if (lane == 0) {
            refill_ok = mbar_wait(&empty[st], (c / STAGES) & 1);
            if (refill_ok) {
              issue(c + STAGES);
              ++issued;
            }
          }
          if (!__shfl_sync(0xffffffffu, refill_ok ? 1 : 0, 0)) {
            record_status(kDevTimeout);
            ok = false;
          }
        }
      }
    };
    // Each warp stores its own normalised sub-partial (A, L = ln Z) of its 16 rows
    // and key share into `dst` ([WN][TR][kPStride], then [WN][TR]).
    auto close = [&](float* dst) {
      float z[2];
      z[0] = quad_sum(acc.l[0]);
      z[1] = quad_sum(acc.l[1]);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = 16 * wm + (lane >> 2) + 8 * i;
        const float inv = z[i] > 0.f ? 1.f / z[i] : 0.f;
        float* row = dst + (wn * TR + r) * C::kPStride;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
          *reinterpret_cast<float2*>(row + n * 8 + 2 * (lane & 3)) =
              make_float2(acc.o[n][2 * i] * inv, acc.o[n][2 * i + 1] * inv);
        if ((lane & 3) == 0) dst[C::kPartL + wn * TR + r] = z[i] > 0.f ? (acc.m[i] + log2f(z[i])) * kLn2 : kNegInf;
      }
      acc.reset();
    };
    auto drain = [&]() {  // copies issued but never consumed (after a timeout) land first
      if (tid == 0 && !ok) {
        for (int c = max(0, issued - STAGES); c < issued; ++c)
          if (!mbar_wait(&full[c % STAGES], (c / STAGES) & 1)) record_status(kDevTimeout);
      }
    };

    // -------------------------------------------------------- the two segments
    if (has_in) {
      run(0, nA);
      close(in_part);
    }
    if (has_out) {
      run(nA, n_local);
      drain();
      __syncthreads();  // every warp is done with the ring before it holds the partial
      close(out_part);
    } else {
      drain();
    }

    // -------------------------------------------------------- merge
    constexpr int kC4 = D / 4;  // float4 columns of a row
    // Step 1, in place: each partial this CTA holds becomes one partial per row
    // (its WN key-share sub-partials combined into sub-partial 0).
    __syncthreads();
    auto fold = [&](float* part) {
      for (int item = tid; item < nrows * kC4; item += C::kThreads) {
        const int r = item / kC4;
        const int c4 = (item % kC4) * 4;
        float l2[WN];
        float4 a[WN];
#pragma unroll
        for (int w = 0; w < WN; ++w) {
          l2[w] = part[C::kPartL + w * TR + r] * kLog2e;
          a[w] = *reinterpret_cast<const float4*>(part + (w * TR + r) * C::kPStride + c4);
        }
        float4 o;
        const float lse2 = lse2_combine<WN>(l2, a, o);
        // The items of a row are consecutive lanes of one warp (kC4 divides 32):
        // they have all read the row's L values before one of them rewrites them.
        __syncwarp(__activemask());
        *reinterpret_cast<float4*>(part + r * C::kPStride + c4) = o;
        if (c4 == 0) part_l_fold(part, C::kPartL, r, lse2);
      }
    };
    if (WN > 1 && cluster_mode) {  // cluster merges read one partial per CTA
      if (has_in) fold(in_part);
      if (has_out) fold(out_part);
    }
    cp_async_wait_all();
    if (cluster_mode) {
      cluster_sync();
    } else {
      __syncthreads();
    }
    if (merger) {
      const int rp = cluster_mode ? (nrows + S - 1) / S : nrows;
      const int r_lo = cluster_mode ? split * rp : 0;
      const int r_hi = min(nrows, r_lo + rp);
      const uint32_t out_a = smem_u32(out_part);
      const uint32_t in_a = smem_u32(in_part);
      uint32_t owners = 0;  // CTAs holding a prefix partial
      for (int s2 = 0; s2 < S; ++s2) {
        int a0, a1;
        prefix_range(s2, S, out_chunks, in_chunks, a0, a1);
        if (a1 > a0) owners |= 1u << s2;
      }
      auto ld_f = [&](uint32_t base, int rank, int f) -> float {
        const uint32_t ad = base + f * 4;
        return cluster_mode ? ld_dsmem_f32(dsmem_addr(ad, rank)) : ld_shared_f32(ad);
      };
      auto ld_f4 = [&](uint32_t base, int rank, int f) -> float4 {
        const uint32_t ad = base + f * 4;
        return cluster_mode ? ld_dsmem_f4(dsmem_addr(ad, rank)) : ld_shared_f4(ad);
      };
      const int n_items = (r_hi - r_lo) * kC4;
      // Entries of a row: prefix entry k is the folded partial of CTA k (cluster
      // mode) or this CTA's key-share sub-partial k; block entry w likewise
      // (folded partial of the last CTA in cluster mode, sub-partial w otherwise).
      constexpr int kOutE = kMaxSplits;
      constexpr int kInE = WN;
      const int n_out_e = cluster_mode ? S : WN;
      const int n_in_e = cluster_mode ? 1 : WN;
      // Phase W, one thread per row: every weight of the row and where it goes.
      // Row slot (kWt floats): [0,kOutE) prefix weights, [kOutE,+kInE) block weights
      // (already scaled by the block's share of A_full), then wo (A_out's share of
      // A_full), L_out, L_full (or L_in), kind, cache entry, output entry.
      float* wt = reinterpret_cast<float*>(q_s);  // the Q tile is dead by now
      constexpr int kWt = kOutE + kInE + 6;
      for (int r = r_lo + tid; r < r_hi; r += C::kThreads) {
        float* wr = wt + (r - r_lo) * kWt;
        const int pos = s_pos[r];
        const int rho = row0 + r;
        const int j = rho % g;
        float kind = 0.f;
        float lo2 = kNegInf, li2 = kNegInf;
        // the block partial's normalisers first: their loads go out with the prefix's
        float l2i[kInE];
#pragma unroll
        for (int w = 0; w < kInE; ++w) {
          l2i[w] = kNegInf;
          if (p.do_in && pos >= 0 && w < n_in_e)
            l2i[w] = (cluster_mode ? ld_f(in_a, S - 1, C::kPartL + r) : in_part[C::kPartL + w * TR + r]) * kLog2e;
        }
        if (pos >= 0) {
          const int ce = (in0 + pos) * p.hq + hk * g + j;
          wr[kOutE + kInE + 4] = __int_as_float(ce);
          wr[kOutE + kInE + 5] = __int_as_float((q0 + rho / g) * p.hq + hk * g + j);
          if (do_out && s_rec[j]) {
            float l2[kOutE];
#pragma unroll
            for (int k = 0; k < kOutE; ++k) {
              l2[k] = kNegInf;
              if (k < n_out_e && (owners >> (cluster_mode ? k : 0) & 1u))
                l2[k] = (cluster_mode ? ld_f(out_a, k, C::kPartL + r) : out_part[C::kPartL + k * TR + r]) * kLog2e;
            }
            lo2 = log2_weights<kOutE>(l2, wr);
            kind = 1.f;
          } else if (p.fused) {
            lo2 = (C::kStageCache ? cache_s[TR * C::kPStride + r] : p.cache_l[ce]) * kLog2e;
            kind = 2.f;
          } else {
            kind = 3.f;  // block pass alone
          }
          if (p.do_in) li2 = log2_weights<kInE>(l2i, wr + kOutE);
        }
        float wo = 1.f, lf2 = li2;
        if (p.fused && pos >= 0) {
          const float m2 = fmaxf(lo2, li2);
          wo = 0.f;
          float wi = 0.f;
          lf2 = kNegInf;
          if (m2 != kNegInf) {
            wo = lo2 == kNegInf ? 0.f : ex2(lo2 - m2);
            wi = li2 == kNegInf ? 0.f : ex2(li2 - m2);
            const float inv = rcp_approx(wo + wi);
            lf2 = m2 + lg2_approx(wo + wi);
            wo *= inv;
            wi *= inv;
          }
#pragma unroll
          for (int w = 0; w < kInE; ++w) wr[kOutE + w] *= wi;
        }
        wr[kOutE + kInE + 0] = wo;
        wr[kOutE + kInE + 1] = lo2 == kNegInf ? kNegInf : lo2 * kLn2;
        wr[kOutE + kInE + 2] = lf2 == kNegInf ? kNegInf : lf2 * kLn2;
        wr[kOutE + kInE + 3] = kind;
      }
      __syncthreads();
      // Phase C, (row, 4 columns) items: loads and multiply-adds only.
      for (int item = tid; item < n_items; item += C::kThreads) {
        const int r = r_lo + item / kC4;
        const int c4 = (item % kC4) * 4;
        const float* wr = wt + (r - r_lo) * kWt;
        const int kind = static_cast<int>(wr[kOutE + kInE + 3]);
        if (kind == 0) continue;
        const size_t ce = static_cast<unsigned>(__float_as_int(wr[kOutE + kInE + 4]));
        const size_t fe = static_cast<unsigned>(__float_as_int(wr[kOutE + kInE + 5]));
        // every load of the item is issued before its stores (a load after a
        // store to a generic address would wait for it)
        float4 vi[kInE];
        if (p.do_in) {
#pragma unroll
          for (int w = 0; w < kInE; ++w) {
            if (w >= n_in_e) continue;
            vi[w] = cluster_mode ? ld_f4(in_a, S - 1, r * C::kPStride + c4)
                                 : *reinterpret_cast<const float4*>(in_part + (w * TR + r) * C::kPStride + c4);
          }
        }
        float4 ao = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kind == 1) {
          float4 v[kOutE];
#pragma unroll
          for (int k = 0; k < kOutE; ++k) {
            if (wr[k] == 0.f) continue;
            v[k] = cluster_mode ? ld_f4(out_a, k, r * C::kPStride + c4)
                                : *reinterpret_cast<const float4*>(out_part + (k * TR + r) * C::kPStride + c4);
          }
#pragma unroll
          for (int k = 0; k < kOutE; ++k)
            if (wr[k] != 0.f) fma4(ao, wr[k], v[k]);
        } else if (kind == 2) {
          ao = C::kStageCache ? *reinterpret_cast<const float4*>(cache_s + r * C::kPStride + c4)
                              : *reinterpret_cast<const float4*>(p.cache_a + ce * D + c4);
        }
        float4 ai = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.do_in) {
#pragma unroll
          for (int w = 0; w < kInE; ++w)
            if (w < n_in_e) fma4(ai, wr[kOutE + w], vi[w]);
        }
        if (kind == 1) {
          *reinterpret_cast<float4*>(p.cache_a + ce * D + c4) = ao;
          if (c4 == 0) p.cache_l[ce] = wr[kOutE + kInE + 1];
        }
        if (!p.do_in) continue;
        if (!p.fused) {
          *reinterpret_cast<float4*>(p.a_in + fe * D + c4) = ai;
          if (c4 == 0) p.l_in[fe] = wr[kOutE + kInE + 2];
          continue;
        }
        const float wo = wr[kOutE + kInE + 0];
        __nv_bfloat16* dst = p.a_full + fe * D + c4;
        *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(fmaf(wo, ao.x, ai.x), fmaf(wo, ao.y, ai.y));
        *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(fmaf(wo, ao.z, ai.z), fmaf(wo, ao.w, ai.w));
        if (c4 == 0 && p.l_full) p.l_full[fe] = wr[kOutE + kInE + 2];
      }
    }
    if (cluster_mode) cluster_sync();  // no CTA leaves while its partials may still be read
  }

  // ------------------------------------------------------------ cache-state epilogue
  if (need_state) state_epilogue(p, tid, C::kThreads, &s_flag);
}

// ------------------------------------------------------------------ similarity gate

struct SimParams {
  int hq, d, total_q, total_in;
  const int* cu_q;
  const int* q_rows;
  const int* cu_in;
  const __nv_bfloat16* q;
  const __nv_bfloat16* q_ref;
  float* cos_out;
};

// cos(Q_bh, q_ref_bh) over the active rows x d of (b, h); one CTA per (b, h).
// Fixed order: each thread accumulates a fixed strided subset, then a fixed tree.
__global__ void __launch_bounds__(256) similarity_kernel(const SimParams p) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x / p.hq;
  const int h = blockIdx.x % p.hq;
  const int q0 = p.cu_q[b];
  const int R = p.cu_q[b + 1] - q0;
  const int in0 = p.cu_in[b];
  const int n_in = p.cu_in[b + 1] - in0;
  const int vpr = p.d / 8;
  float dot = 0.f, nx = 0.f, ny = 0.f;
  const bool ranges_ok = q0 >= 0 && R >= 0 && q0 + R <= p.total_q && in0 >= 0 && n_in >= 0 && in0 + n_in <= p.total_in;
  if (!ranges_ok && threadIdx.x == 0) record_status(kDevBadIndex);
  for (int v = threadIdx.x; ranges_ok && v < R * vpr; v += 256) {
    const int r = v / vpr;
    const int c = v % vpr;
    const int prow = q0 + r;
    const int pos = p.q_rows ? p.q_rows[prow] : r;
    if (pos < 0 || pos >= n_in) {
      record_status(kDevBadIndex);
      continue;
    }
    const uint4 xv = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(prow) * p.hq + h) * p.d + c * 8);
    const uint4 yv =
        *reinterpret_cast<const uint4*>(p.q_ref + (static_cast<size_t>(in0 + pos) * p.hq + h) * p.d + c * 8);
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
    const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&yv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 xf = __bfloat1622float2(x2[e]);
      const float2 yf = __bfloat1622float2(y2[e]);
      dot = fmaf(xf.x, yf.x, dot);
      dot = fmaf(xf.y, yf.y, dot);
      nx = fmaf(xf.x, xf.x, nx);
      nx = fmaf(xf.y, xf.y, nx);
      ny = fmaf(yf.x, yf.x, ny);
      ny = fmaf(yf.y, yf.y, ny);
    }
  }
  __shared__ float red[3][8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, off);
    nx += __shfl_xor_sync(0xffffffffu, nx, off);
    ny += __shfl_xor_sync(0xffffffffu, ny, off);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = dot;
    red[1][w] = nx;
    red[2][w] = ny;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sd = 0.f, sx = 0.f, sy = 0.f;
    for (int i = 0; i < 8; ++i) {
      sd += red[0][i];
      sx += red[1][i];
      sy += red[2][i];
    }
    const float den = sqrtf(sx) * sqrtf(sy);
    p.cos_out[blockIdx.x] = den > 0.f ? sd / den : 0.f;
  }
}

// ------------------------------------------------------------------ branch hooks

struct CacheCopyParams {
  int hq, d, num_seqs, total_in, src, dst;
  const int* cu_in;
  float* a_out;
  float* l_out;
  uint8_t* valid;
  __nv_bfloat16* q_ref;
  int* m_acc;
};

// Entries of block positions 0..min(B_src, B_dst)-1 from sequence src to dst
// (grid-stride over (position, head, 4 columns) items); block 0 also copies the
// per-head validity and counts.
__global__ void __launch_bounds__(256) cache_copy_kernel(const CacheCopyParams p) {
  pdl_wait();
  pdl_trigger();
  const int s0 = p.cu_in[p.src], s1 = p.cu_in[p.src + 1];
  const int d0 = p.cu_in[p.dst], d1 = p.cu_in[p.dst + 1];
  if (s0 < 0 || s1 < s0 || s1 > p.total_in || d0 < 0 || d1 < d0 || d1 > p.total_in) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(kDevBadIndex);
    return;
  }
  const int n = min(s1 - s0, d1 - d0);
  const int c4 = p.d / 4;
  const long items = static_cast<long>(n) * p.hq * c4;
  for (long it = blockIdx.x * 256l + threadIdx.x; it < items; it += static_cast<long>(gridDim.x) * 256) {
    const long e = it / c4;  // (position, head)
    const int c = static_cast<int>(it % c4) * 4;
    const long se = static_cast<long>(s0) * p.hq + e, de = static_cast<long>(d0) * p.hq + e;
    *reinterpret_cast<float4*>(p.a_out + de * p.d + c) = *reinterpret_cast<const float4*>(p.a_out + se * p.d + c);
    if (p.q_ref)
      *reinterpret_cast<uint2*>(p.q_ref + de * p.d + c) = *reinterpret_cast<const uint2*>(p.q_ref + se * p.d + c);
    if (c == 0) p.l_out[de] = p.l_out[se];
  }
  if (blockIdx.x == 0) {
    const bool filled = d1 - d0 <= s1 - s0;
    for (int h = threadIdx.x; h < p.hq; h += 256) {
      p.valid[p.dst * p.hq + h] = filled ? p.valid[p.src * p.hq + h] : 0;
      if (p.m_acc) p.m_acc[p.dst * p.hq + h] = p.m_acc[p.src * p.hq + h];
    }
  }
}

struct InvalidateParams {
  int hq, num_seqs;
  const uint8_t* mask;
  uint8_t* valid;
  int* m_acc;
};

__global__ void __launch_bounds__(256) cache_invalidate_kernel(const InvalidateParams p) {
  pdl_wait();
  pdl_trigger();
  const int total = p.num_seqs * p.hq;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < total; i += gridDim.x * 256) {
    if (p.mask && !p.mask[i / p.hq]) continue;
    p.valid[i] = 0;
    if (p.m_acc) p.m_acc[i] = 0;
  }
}

// ------------------------------------------------------------------ element-wise merge

struct MergeParams {
  int64_t n;
  int d;
  const float* a_out;
  const float* l_out;
  const float* a_in;
  const float* l_in;
  float* a_f32;
  __nv_bfloat16* a_bf16;
  float* l_full;
};

__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t total = p.n * p.d;
  for (int64_t idx = blockIdx.x * 256ll + threadIdx.x; idx < total; idx += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t e = idx / p.d;
    const int col = static_cast<int>(idx % p.d);
    const float lo = p.l_out[e];
    const float li = p.l_in[e];
    const float mx = fmaxf(lo, li);
    float a = 0.f;
    float l = kNegInf;
    if (mx != kNegInf) {
      const float wo = lo == kNegInf ? 0.f : expf(lo - mx);
      const float wi = li == kNegInf ? 0.f : expf(li - mx);
      const float den = wo + wi;
      a = (wo * p.a_out[idx] + wi * p.a_in[idx]) / den;
      l = mx + logf(den);
    }
    if (p.a_f32) p.a_f32[idx] = a;
    if (p.a_bf16) p.a_bf16[idx] = __float2bfloat16_rn(a);
    if (col == 0 && p.l_full) p.l_full[e] = l;
  }
}

}  // namespace fb
