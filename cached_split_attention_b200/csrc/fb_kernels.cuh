// FlashBlock denoise-step attention kernels (sm_100a).
//
// One kernel, `attn_kernel`, serves the out-of-block pass, the in-block pass and
// the fused step.  Its grid holds two kinds of CTAs:
//
//   in-CTAs   one per group (sequence b, kv-head hk, row tile t): softmax
//             attention of the tile's rows over the block's keys J_in(b);
//   out-CTAs  `splits` per group: attention over one key range of the prefix
//             J_out(b), only for groups with a head that recomputes.
//
// A "row" of a group is a (query token, q-head of the kv-head's group) pair, so a
// grouped-query kv-head streams its K/V once for all its q-heads.  Every CTA
// produces a partial (A, L) for its rows: A normalised, L = ln Z (FlashBlock,
// "Mecanismo Central").  Partials reach global memory; the last CTA of a group to
// finish (an atomic counter, no waiting) combines them with the log-space rule
//   A = sum_s e^{L_s-m} A_s / sum_s e^{L_s-m},  L = m + ln sum_s e^{L_s-m},
// which is associative, so splitting the prefix and merging the block partial
// are the same operation.  It stores the recomputed out-of-block partial in the
// cache, reads the cached one for heads that reuse, and writes A_full / L_full.
// The last CTA of the whole grid marks recomputed heads valid and writes the
// decision mask.  No CTA ever waits for another one.
//
// Inside a CTA: thread 0 streams K/V key tiles with TMA (128-byte swizzle,
// evict-first L2 policy) through a ring of mbarrier-guarded stages; the WM x WN
// warps run mma.sync m16n8k16 (bf16 in, fp32 accumulate) with an online softmax
// in base 2.  Warp (wm, wn) owns 16 rows and
// a 1/WN share of every key tile; the WN shares are merged through shared memory.
#pragma once

#include <limits>

#include "fb_device.cuh"

namespace fb {

constexpr unsigned kGateTau = 1u, kGateHead = 2u, kForceRecompute = 4u, kForceReuse = 8u;
constexpr int kBN = 64;      // keys per pipeline stage
constexpr int kStages = 4;   // pipeline depth
constexpr int kMaxGroup = 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -std::numeric_limits<float>::infinity();

__device__ int g_status;  // first error recorded by any kernel (0 = none)

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

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
  int tr, tiles, n_groups, splits, kps, slots, n_in_ctas;
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
  __nv_bfloat16* q_ref;
  __nv_bfloat16* a_full;
  float* l_full;
  uint8_t* decision_out;
  float* a_in;
  float* l_in;
  // workspace
  float* part_a;
  float* part_l;
  int* group_ctr;
  int* grid_ctr;
};

// Reuse decision of (b, h); see fb_step in flashblock.h.
__device__ __forceinline__ bool head_recompute(const Params& p, int b, int h) {
  const int idx = b * p.hq + h;
  if (!p.update_state) return p.head_mask ? (p.head_mask[idx] != 0) : true;
  if (p.flags & kForceRecompute) return true;
  if (!p.valid[idx]) return true;
  if (p.flags & kForceReuse) return false;
  if (p.head_reuse_in) return p.head_reuse_in[idx] == 0;
  bool reuse = true;
  if (p.flags & kGateTau) reuse = reuse && (p.n_updated[b] < p.tau);
  if (p.flags & kGateHead) reuse = reuse && (p.cos[idx] > p.gamma);
  return !reuse;
}

template <int D, int WM, int WN>
struct Cfg {
  static constexpr int kRows = 16 * WM;
  static constexpr int kConsumerWarps = WM * WN;
  static constexpr int kThreads = kConsumerWarps * 32;
  static constexpr int kKW = kBN / WN;              // keys per warp per stage
  static constexpr int kTileBytes = kBN * D * 2;    // K (or V) tile of one stage
  static constexpr int kHalfBytes = kBN * 128;      // one 64-column swizzle span
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStageArea = kStages * kStageBytes;
  static constexpr int kQStride = D + 8;            // padded Q row, elements
  static constexpr int kQBytes = kRows * kQStride * 2;
  static constexpr int kScratchBytes = WN > 1 ? kConsumerWarps * (D / 2 + 4) * 32 * 4 : 0;
  static constexpr int kSmem = 1024 + kStageArea + kQBytes + 2 * kStages * 8;
  static_assert(kKW % 16 == 0, "keys per warp must be a multiple of 16");
  static_assert(kScratchBytes <= kStageArea, "combine scratch must fit in the stage ring");
  static_assert(D == 64 || D == 128, "head_dim");
};

// Byte offset of (key row kr, column dd) inside a stage tile written by TMA with
// 128-byte swizzle: 16-byte chunk c of a 128-byte row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int kr, int dd) {
  return static_cast<uint32_t>((dd >> 6) * (kBN * 128) + kr * 128 + ((((dd & 63) >> 3) ^ (kr & 7)) << 4));
}

template <int D, int WM, int WN>
__global__ void __launch_bounds__(Cfg<D, WM, WN>::kThreads, 1) attn_kernel(const __grid_constant__ Params p) {
  using C = Cfg<D, WM, WN>;
  constexpr int TR = C::kRows;
  constexpr int KW = C::kKW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  __nv_bfloat16* q_s = reinterpret_cast<__nv_bfloat16*>(smem + C::kStageArea);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStageArea + C::kQBytes);
  uint64_t* empty = full + kStages;
  __shared__ uint8_t s_rec[kMaxGroup];
  __shared__ int s_flag;
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---------------------------------------------------------------- role
  const int cta = blockIdx.x;
  const bool is_in = cta < p.n_in_ctas;
  int gidx, split;
  if (is_in) {
    gidx = cta;
    split = p.splits;  // the block partial uses the last slot of the group
  } else {
    const int o = cta - p.n_in_ctas;
    gidx = o / p.splits;
    split = o % p.splits;
  }
  const int t = gidx % p.tiles;
  const int bh = gidx / p.tiles;
  const int hk = bh % p.hkv;
  const int b = bh / p.hkv;
  const int g = p.g;

  const int q0 = p.cu_q[b];
  const int rows = (p.cu_q[b + 1] - q0) * g;
  const int row0 = t * TR;
  const int nrows = min(TR, rows - row0);
  const int out0 = p.cu_out[b];
  const int n_out = p.cu_out[b + 1] - out0;
  const int in0 = p.cu_in[b];
  const int n_in = p.cu_in[b + 1] - in0;
  const int n_out_splits = n_out > 0 ? (n_out + p.kps - 1) / p.kps : 1;
  // Offsets that do not fit the buffers the host described: record and do nothing.
  const bool ranges_ok = q0 >= 0 && rows >= 0 && q0 + rows / max(g, 1) <= p.total_q && out0 >= 0 && n_out >= 0 &&
                         out0 + n_out <= p.total_out && in0 >= 0 && n_in >= 0 && in0 + n_in <= p.total_in &&
                         rows / max(g, 1) <= n_in;
  if (!ranges_ok && tid == 0 && t == 0 && split == 0) record_status(kDevBadIndex);

  if (tid < g) s_rec[tid] = head_recompute(p, b, hk * g + tid) ? 1 : 0;
  if (tid == 0) s_abort = 0;
  __syncthreads();
  bool any_rec = false;
  for (int j = 0; j < g; ++j) any_rec |= (s_rec[j] != 0);

  const int expected = (p.do_out && any_rec ? n_out_splits : 0) + (p.fused ? 1 : 0);
  int k_lo, k_hi;
  bool work;
  if (is_in) {
    k_lo = 0;
    k_hi = n_in;
    work = ranges_ok && p.do_in && nrows > 0;
  } else {
    k_lo = split * p.kps;
    k_hi = min(n_out, k_lo + p.kps);
    work = ranges_ok && p.do_out && nrows > 0 && any_rec && split < n_out_splits;
  }
  const bool counted = work && (p.fused || !is_in);  // reaches the group counter

  if (work) {
    // ------------------------------------------------------------ Q tile
    for (int v = tid; v < TR * (D / 8); v += C::kThreads) {
      const int r = v / (D / 8);
      const int c = v % (D / 8);
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (r < nrows) {
        const int rho = row0 + r;
        const int it = rho / g;
        const int h = hk * g + rho % g;
        val = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(q0 + it) * p.hq + h) * D + c * 8);
      }
      *reinterpret_cast<uint4*>(q_s + r * C::kQStride + c * 8) = val;
    }
    if (tid == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], C::kConsumerWarps);
      }
      fence_barrier_init();
    }
    __syncthreads();

    const int n_chunks = k_hi > k_lo ? (k_hi - k_lo + kBN - 1) / kBN : 0;

    // Thread 0 issues the TMA copies: the first kStages chunks now, chunk c + kStages
    // once every warp has released stage c % kStages.
    const CUtensorMap* tk = is_in ? &p.tm_k_in : &p.tm_k_out;
    const CUtensorMap* tv = is_in ? &p.tm_v_in : &p.tm_v_out;
    const int y0 = (is_in ? in0 : out0) + k_lo;
    uint64_t pol = 0;
    int issued = 0;
    auto issue = [&](int c) {
      const int st = c % kStages;
      mbar_arrive_expect_tx(&full[st], C::kStageBytes);
      uint8_t* kd = stages + st * C::kStageBytes;
      uint8_t* vd = kd + C::kTileBytes;
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_2d(kd + hh * C::kHalfBytes, tk, &full[st], hk * D + hh * 64, y0 + c * kBN, pol);
        tma_load_2d(vd + hh * C::kHalfBytes, tv, &full[st], hk * D + hh * 64, y0 + c * kBN, pol);
      }
      ++issued;
    };
    if (tid == 0 && n_chunks > 0) {
      prefetch_tensormap(tk);
      prefetch_tensormap(tv);
      pol = l2_policy_evict_first();
      for (int c = 0; c < min(kStages, n_chunks); ++c) issue(c);
    }
    {
      // ---------------------------------------------------------- consumers
      const int wm = warp % WM;
      const int wn = warp / WM;
      const bool rows_active = 16 * wm < nrows;
      uint32_t qf[D / 16][4];
      if (rows_active) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ldsm_x4(qf[kk], smem_u32(q_s + (16 * wm + (lane & 15)) * C::kQStride + kk * 16 + (lane >> 4) * 8));
      }
      float o[D / 8][4];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      float m_run[2] = {kNegInf, kNegInf};
      float l_run[2] = {0.f, 0.f};
      bool ok = true;

      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStages;
        if (!mbar_wait(&full[st], (c / kStages) & 1)) {
          record_status(kDevTimeout);
          s_abort = 1;
          ok = false;
          break;
        }
        if (rows_active) {
          const uint32_t kb = smem_u32(stages + st * C::kStageBytes);
          const uint32_t vb = kb + C::kTileBytes;
          float s[KW / 8][4];
#pragma unroll
          for (int n = 0; n < KW / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
          // S = Q K^T over this warp's KW keys
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int nb = 0; nb < KW / 16; ++nb) {
              const int mi = lane >> 3;
              const int kr = wn * KW + nb * 16 + (mi >> 1) * 8 + (lane & 7);
              const int dd = kk * 16 + (mi & 1) * 8;
              uint32_t r[4];
              ldsm_x4(r, kb + swz(kr, dd));
              mma_bf16_16816(s[2 * nb], qf[kk], r[0], r[1]);
              mma_bf16_16816(s[2 * nb + 1], qf[kk], r[2], r[3]);
            }
          }
          // scale to base 2, mask keys past the range end
          const int key0 = k_lo + c * kBN + wn * KW;
          const bool need_mask = key0 + KW > k_hi;
#pragma unroll
          for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float v = s[n][e] * p.scale_log2;
              if (need_mask && key0 + n * 8 + 2 * (lane & 3) + (e & 1) >= k_hi) v = kNegInf;
              s[n][e] = v;
            }
          }
          // online softmax
          float mx[2] = {m_run[0], m_run[1]};
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
            alpha[i] = ex2(m_run[i] - msafe[i]);
            m_run[i] = mx[i];
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
          l_run[0] = l_run[0] * alpha[0] + rs[0];
          l_run[1] = l_run[1] * alpha[1] + rs[1];
#pragma unroll
          for (int n = 0; n < D / 8; ++n) {
            o[n][0] *= alpha[0];
            o[n][1] *= alpha[0];
            o[n][2] *= alpha[1];
            o[n][3] *= alpha[1];
          }
          // O += P V
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
              const int kr = wn * KW + kb2 * 16 + (mi & 1) * 8 + (lane & 7);
              const int dd = np * 16 + (mi >> 1) * 8;
              uint32_t r[4];
              ldsm_x4_t(r, vb + swz(kr, dd));
              mma_bf16_16816(o[2 * np], a, r[0], r[1]);
              mma_bf16_16816(o[2 * np + 1], a, r[2], r[3]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (tid == 0 && c + kStages < n_chunks) {
          if (!mbar_wait(&empty[st], (c / kStages) & 1)) {
            record_status(kDevTimeout);
            s_abort = 1;
            ok = false;
            break;
          }
          issue(c + kStages);
        }
      }
      // Drain: copies issued but never consumed (only after a timeout) land first.
      if (tid == 0 && !ok) {
        for (int c = max(0, issued - kStages); c < issued; ++c)
          if (!mbar_wait(&full[c % kStages], (c / kStages) & 1)) record_status(kDevTimeout);
      }

      l_run[0] = quad_sum(l_run[0]);
      l_run[1] = quad_sum(l_run[1]);

      // ---------------------------------------------------- merge the WN shares
      if constexpr (WN > 1) {
        __syncthreads();
        const bool aborted = s_abort != 0;
        float* scr = reinterpret_cast<float*>(stages);
        constexpr int kRegs = D / 2 + 4;
        float* mine = scr + (wn * WM + wm) * kRegs * 32;
        if (!aborted && wn > 0) {
#pragma unroll
          for (int n = 0; n < D / 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) mine[(n * 4 + e) * 32 + lane] = o[n][e];
          mine[(D / 2 + 0) * 32 + lane] = m_run[0];
          mine[(D / 2 + 1) * 32 + lane] = m_run[1];
          mine[(D / 2 + 2) * 32 + lane] = l_run[0];
          mine[(D / 2 + 3) * 32 + lane] = l_run[1];
        }
        __syncthreads();
        if (!aborted && wn == 0) {
#pragma unroll 1
          for (int w2 = 1; w2 < WN; ++w2) {
            const float* th = scr + (w2 * WM + wm) * kRegs * 32;
            float a1[2], a2[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const float m2 = th[(D / 2 + i) * 32 + lane];
              const float l2 = th[(D / 2 + 2 + i) * 32 + lane];
              const float mn = fmaxf(m_run[i], m2);
              const float ms = mn == kNegInf ? 0.f : mn;
              a1[i] = ex2(m_run[i] - ms);
              a2[i] = ex2(m2 - ms);
              l_run[i] = l_run[i] * a1[i] + l2 * a2[i];
              m_run[i] = mn;
            }
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
              o[n][0] = o[n][0] * a1[0] + th[(n * 4 + 0) * 32 + lane] * a2[0];
              o[n][1] = o[n][1] * a1[0] + th[(n * 4 + 1) * 32 + lane] * a2[0];
              o[n][2] = o[n][2] * a1[1] + th[(n * 4 + 2) * 32 + lane] * a2[1];
              o[n][3] = o[n][3] * a1[1] + th[(n * 4 + 3) * 32 + lane] * a2[1];
            }
          }
        }
      }

      // ---------------------------------------------------- write the partial
      if (ok && wn == 0 && rows_active) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = 16 * wm + (lane >> 2) + 8 * i;
          if (r < nrows) {
            const float l = l_run[i];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float lnat = l > 0.f ? (m_run[i] + log2f(l)) * kLn2 : kNegInf;
            float* arow;
            float* lptr;
            if (is_in && !p.fused) {
              const int rho = row0 + r;
              const size_t e = static_cast<size_t>(q0 + rho / g) * p.hq + hk * g + rho % g;
              arow = p.a_in + e * D;
              lptr = p.l_in + e;
            } else {
              const size_t e = (static_cast<size_t>(gidx) * p.slots + split) * TR + r;
              arow = p.part_a + e * D;
              lptr = p.part_l + e;
            }
#pragma unroll
            for (int n = 0; n < D / 8; ++n)
              *reinterpret_cast<float2*>(arow + n * 8 + 2 * (lane & 3)) =
                  make_float2(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
            if ((lane & 3) == 0) *lptr = lnat;
          }
        }
      }
    }

    // q_ref follows the queries of heads that recompute (in-CTA of fb_step)
    if (is_in && p.fused && p.q_ref != nullptr) {
      for (int v = tid; v < nrows * (D / 8); v += C::kThreads) {
        const int r = v / (D / 8);
        const int c = v % (D / 8);
        const int rho = row0 + r;
        const int j = rho % g;
        if (!s_rec[j]) continue;
        const int prow = q0 + rho / g;
        const int pos = p.q_rows ? p.q_rows[prow] : rho / g;
        if (pos < 0 || pos >= n_in) {
          record_status(kDevBadIndex);
          continue;
        }
        const size_t e = (static_cast<size_t>(in0 + pos) * p.hq + hk * g + j) * D + c * 8;
        *reinterpret_cast<uint4*>(p.q_ref + e) = *reinterpret_cast<const uint4*>(q_s + r * C::kQStride + c * 8);
      }
    }
  }

  // ---------------------------------------------------------------- group merge
  if (counted) {
    __threadfence();
    __syncthreads();
    if (tid == 0) s_flag = (atomicAdd(&p.group_ctr[gidx], 1) == expected - 1) ? 1 : 0;
    __syncthreads();
    if (s_flag) {
      __threadfence();
      constexpr int VPT = D / 32;  // floats per lane of one row
      const int nw = C::kThreads / 32;
      for (int r = warp; r < nrows; r += nw) {
        const int rho = row0 + r;
        const int it = rho / g;
        const int j = rho % g;
        const int h = hk * g + j;
        const int prow = q0 + it;
        const int pos = p.q_rows ? p.q_rows[prow] : it;
        if (pos < 0 || pos >= n_in) {
          record_status(kDevBadIndex);
          continue;
        }
        const size_t ce = static_cast<size_t>(in0 + pos) * p.hq + h;
        float ao[VPT];
        float lo = kNegInf;
#pragma unroll
        for (int v = 0; v < VPT; ++v) ao[v] = 0.f;
        const bool rec = s_rec[j] != 0;
        if (p.do_out && rec) {
          const size_t base = static_cast<size_t>(gidx) * p.slots * TR + r;
          float mx = kNegInf;
          for (int s2 = 0; s2 < n_out_splits; ++s2) mx = fmaxf(mx, __ldcg(p.part_l + base + s2 * TR));
          if (mx != kNegInf) {
            float den = 0.f;
            for (int s2 = 0; s2 < n_out_splits; ++s2) {
              const float ls = __ldcg(p.part_l + base + s2 * TR);
              const float w = ls == kNegInf ? 0.f : expf(ls - mx);
              den += w;
              const float* src = p.part_a + (base + s2 * TR) * D + lane * VPT;
#pragma unroll
              for (int v = 0; v < VPT; ++v) ao[v] += w * __ldcg(src + v);
            }
            const float inv = 1.f / den;
#pragma unroll
            for (int v = 0; v < VPT; ++v) ao[v] *= inv;
            lo = mx + logf(den);
          }
#pragma unroll
          for (int v = 0; v < VPT; ++v) p.cache_a[ce * D + lane * VPT + v] = ao[v];
          if (lane == 0) p.cache_l[ce] = lo;
        } else if (p.fused) {
#pragma unroll
          for (int v = 0; v < VPT; ++v) ao[v] = p.cache_a[ce * D + lane * VPT + v];
          lo = p.cache_l[ce];
        }
        if (p.fused) {
          const size_t ie = (static_cast<size_t>(gidx) * p.slots + p.splits) * TR + r;
          const float li = __ldcg(p.part_l + ie);
          const float* ai = p.part_a + ie * D + lane * VPT;
          const float mx = fmaxf(lo, li);
          float af[VPT];
          float lf = kNegInf;
          if (mx == kNegInf) {
#pragma unroll
            for (int v = 0; v < VPT; ++v) af[v] = 0.f;
          } else {
            const float wo = lo == kNegInf ? 0.f : expf(lo - mx);
            const float wi = li == kNegInf ? 0.f : expf(li - mx);
            const float den = wo + wi;
            const float inv = 1.f / den;
#pragma unroll
            for (int v = 0; v < VPT; ++v) af[v] = (wo * ao[v] + wi * __ldcg(ai + v)) * inv;
            lf = mx + logf(den);
          }
          const size_t fe = static_cast<size_t>(prow) * p.hq + h;
          __nv_bfloat16* dst = p.a_full + fe * D + lane * VPT;
#pragma unroll
          for (int v = 0; v < VPT; v += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + v) = __floats2bfloat162_rn(af[v], af[v + 1]);
          if (lane == 0 && p.l_full) p.l_full[fe] = lf;
        }
      }
      if (tid == 0) p.group_ctr[gidx] = 0;
    }
  }

  // ---------------------------------------------------------------- grid epilogue
  if (p.update_state) {
    __syncthreads();
    __threadfence();
    if (tid == 0) s_flag = (atomicAdd(p.grid_ctr, 1) == static_cast<int>(gridDim.x) - 1) ? 1 : 0;
    __syncthreads();
    if (s_flag) {
      __threadfence();
      const int total = p.num_seqs * p.hq;
      for (int idx = tid; idx < total; idx += C::kThreads) {
        const bool rec = head_recompute(p, idx / p.hq, idx % p.hq);
        if (p.decision_out) p.decision_out[idx] = rec ? 1 : 0;
        if (rec) p.valid[idx] = 1;
      }
      if (tid == 0) *p.grid_ctr = 0;
    }
  }
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
