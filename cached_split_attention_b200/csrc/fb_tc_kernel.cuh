// Tensor-core variant of the FlashBlock attention kernel (sm_100a, tcgen05 + TMEM)
// for head_dim 128 and groups of more than 64 rows: the long-context GQA block
// (32 active tokens x 4 q-heads per kv-head), the video block (1560 tokens per
// head), large varlen branches.
//
// Same decomposition, merge and epilogue as `attn_kernel` (fb_kernels.cuh): a
// group (sequence, kv-head, 128-row tile) is served by a cluster of S CTAs that
// split the prefix chunks; the last CTA also runs the block's chunks; partials
// (A normalised, L = ln Z; FlashBlock, "Mecanismo Central") are combined with the
// log-space merge through distributed shared memory.  What changes is the inner
// loop, per 128-key chunk:
//
//   warp 4R (one thread)    TMA: K chunk -> ring of 3, V chunk -> ring of 3
//   warp 4R+1 (one thread)  S = Q K^T   (tcgen05.mma, M=128 N=128 K=128, fp32 in
//                                        TMEM, two S buffers so the next chunk's S
//                                        overlaps the softmax of this one)
//                           O += P V    (tcgen05.mma with A = P read from TMEM, O in
//                                        TMEM; one O accumulator per segment)
//   warps 0 .. 4R-1         R threads per tile row (= TMEM lane): warp w takes keys
//                           128 (w / 4) / R .. of the rows of lane quarter w % 4.
//                           Each loads its share of the S row and masks it, runs the
//                           max in base 2, P = 2^(s - m) rounded to bf16 and stored
//                           back over S columns already read, and its sum.  O is
//                           rescaled in TMEM only when the running max grows by more
//                           than 2^8 (the stored max may lag: exact, since O and l
//                           always share the same reference).  Three of every eight
//                           2^x go through a cubic on the FMA pipe instead of the
//                           MUFU unit.
//
// R = 1 in a grid that one wave holds, where the stream is bound by HBM.  R = 2
// (the host plan's choice for more CTAs than one wave, e.g. the varlen branches,
// whose later CTAs run with the HBM less loaded): one softmax thread per row is
// bound by its own latencies, and two softmax warps per SM sub-partition fill each
// other's stalls.  The two halves of a row swap their maxima through shared memory
// each chunk (bounded mbarrier handshakes) and add their sums at the end.  R = 2 took
// the varlen branches' recompute call from 82.2 to 73.6 us; on the long-context GQA
// batch (one wave, HBM-bound) it cost 1 % per call.
//
// The MMA thread issues S(c) after P V(c-2) and P V(c) after S(c+1); the tensor
// core runs them in issue order, so S(c+2) never overwrites P(c) before P V(c) has
// read it, and the completion of S(c) implies that of P V(c-2).
//
// Operand layouts in shared memory are the 128-byte-swizzled tiles TMA writes:
// Q and K are K-major (rows of 64-element halves, 8-row groups 1024 bytes apart),
// V is MN-major (key rows of 64 d-columns, the two d-halves 16 KB apart).  P in
// TMEM is K-major: lane = row, 32-bit column j = keys 2j (low half), 2j+1.
//
// TMEM: 512 columns x 128 lanes: S/P buffers at columns 0 and 128, prefix O at
// 256, block O at 384.  Every wait is bounded; on a timeout the CTA records
// kDevTimeout, stops issuing, lets issued copies and MMAs land, and finishes.
#pragma once

#include "fb_kernels.cuh"
#include "fb_tcgen05.cuh"

namespace fb {
namespace tc {

constexpr int kD = 128;
constexpr int kM = 128;           // tile rows = TMEM lanes
constexpr int kN = 128;           // keys per chunk
// Threads of a CTA with R threads per tile row: 4 R row warps, then the TMA warp
// and the MMA warp.
constexpr int threads_for(int row_threads) { return 128 * row_threads + 64; }
constexpr int kHalf = kN * 128;   // 64 columns (128 bytes) x 128 rows: 16 KB
constexpr int kTile = 2 * kHalf;  // 128 x 128 bf16: 32 KB
constexpr int kStages = 3;        // K and V rings
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kStages * kTile;
constexpr int kOffQ = kOffV + kStages * kTile;
constexpr int kOffBar = kOffQ + kTile;
constexpr int kNumBars = 20;
constexpr int kOffPos = kOffBar + kNumBars * 8;
constexpr int kOffMisc = kOffPos + kM * 4;
constexpr int kSmem = 1024 + kOffMisc + 16;  // + alignment of the base to 1024 bytes
// Partials after the pipeline drains (they overlay the K/V rings and P):
// A [kM][kPStride] floats, then L [kM].
constexpr int kPStride = kD + 4;
constexpr int kPartL = kM * kPStride;
constexpr int kPartFloats = kPartL + kM;
constexpr int kOffPartIn = kPartFloats * 4;
// Merge table per row (in the dead Q tile): kMaxSplits prefix weights, the block
// weight, then wo, L_out, L_full (or L_in), kind, cache entry, output entry.
constexpr int kWt = kMaxSplits + 1 + 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColOut = 256;
constexpr uint32_t kColIn = 384;
constexpr uint32_t kIdescS = idesc_bf16(kM, kN, false);
constexpr uint32_t kIdescO = idesc_bf16(kM, kD, true);
constexpr float kRescaleSlack = 8.f;  // log2 units the stored running max may lag
// 2^f on [-1/2, 1/2] by a cubic of least maximum relative error (7.5e-5, far below
// the bf16 rounding of P); fitted by fit_exp2_poly.py beside this file.
constexpr float kExpC0 = 0.9999281167984009f;
constexpr float kExpC1 = 0.6932609677314758f;
constexpr float kExpC2 = 0.24261054396629333f;
constexpr float kExpC3 = 0.05517132207751274f;

static_assert(2 * kPartFloats * 4 <= kOffQ, "both partials fit below the Q tile");
static_assert(kOffPartIn % 16 == 0, "aligned partial");
static_assert(kM * kWt * 4 <= kTile, "merge table fits in the Q tile");
static_assert(kSmem <= 232448, "shared memory per CTA");

// 2^x for a pair of x on the FMA pipe: x = j + f with j = round(x) (the
// 1.5 * 2^23 shifter leaves j in the low mantissa bits of t), 2^f by the cubic,
// 2^j added to the exponent field.  Inputs below -126 give results below 2^-126
// (0 for practical purposes).
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& p0, float& p1) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t shift = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = fadd2(x, shift);
  const uint64_t f = fsub2(x, fsub2(t, shift));
  uint64_t q = ffma2(f2_pack(kExpC3, kExpC3), f, f2_pack(kExpC2, kExpC2));
  q = ffma2(q, f, f2_pack(kExpC1, kExpC1));
  q = ffma2(q, f, f2_pack(kExpC0, kExpC0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

}  // namespace tc

template <int kRowThreads>
__global__ void __launch_bounds__(tc::threads_for(kRowThreads), 1) tc_attn_kernel(const __grid_constant__ Params p) {
  prefetch_maps(p);
  using namespace tc;
  constexpr int kThreads = threads_for(kRowThreads);
  constexpr int kTmaWarp = 4 * kRowThreads;  // warps 0 .. 4R-1 hold the rows
  constexpr int kMmaWarp = kTmaWarp + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* k_full = bars;        // [3] TMA -> MMA
  uint64_t* k_empty = bars + 3;   // [3] MMA -> TMA
  uint64_t* v_full = bars + 6;    // [3]
  uint64_t* v_empty = bars + 9;   // [3]
  uint64_t* s_full = bars + 12;   // [2] MMA -> rows
  uint64_t* p_full = bars + 14;   // rows -> MMA
  uint64_t* pv_done = bars + 15;  // MMA -> rows
  uint64_t* drain = bars + 16;    // MMA -> MMA (all issued MMAs finished)
  int* s_pos = reinterpret_cast<int*>(smem + kOffPos);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* part_out = reinterpret_cast<float*>(smem);
  float* part_in = reinterpret_cast<float*>(smem + kOffPartIn);
  __shared__ uint8_t s_rec[kMaxGroup];
  __shared__ int s_flag;
  __shared__ __align__(8) uint64_t s_lean_bar[2];  // lean path: inputs, cached rows
  // the two softmax warps of a row quarter swap per-row values (the halves' maxima
  // of a chunk, their sums at the end) through s_xv; s_xch: both written, s_xrd:
  // both read (so that a slot is rewritten only after the other warp has read it)
  __shared__ __align__(8) uint64_t s_xch[4], s_xrd[4];
  __shared__ float s_xv[kRowThreads][kRowThreads == 2 ? kM : 1];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.splits;
  const int split = blockIdx.x % S;  // == rank in the cluster
  const int gidx = blockIdx.x / S;
  const int t = gidx % p.tiles;
  const int bh = gidx / p.tiles;
  const int hk = bh % p.hkv;
  const int b = bh / p.hkv;
  const int g = p.g;

  // ------------------------------------------------------------ group metadata
  // Index arrays before the wait for the previous kernel of the stream (see
  // attn_kernel); the cache state after it.
  const int q0 = p.cu_q[b];
  const int n_q = p.cu_q[b + 1] - q0;
  const int out0 = p.cu_out[b];
  const int n_out = p.cu_out[b + 1] - out0;
  const int in0 = p.cu_in[b];
  const int n_in = p.cu_in[b + 1] - in0;
  const bool ranges_ok = q0 >= 0 && n_q >= 0 && q0 + n_q <= p.total_q && out0 >= 0 && n_out >= 0 &&
                         out0 + n_out <= p.total_out && in0 >= 0 && n_in >= 0 && in0 + n_in <= p.total_in &&
                         n_q <= n_in;
  const int row0 = t * kM;
  if (!ranges_ok && tid == 0 && t == 0 && split == 0) record_status(kDevBadIndex);
  const int rows = ranges_ok ? n_q * g : 0;
  const int nrows = max(0, min(kM, rows - row0));
  // Lean reuse path (see attn_kernel).
  LeanRows lr{};
  const LeanSmem<kD> ls(smem, p.reuse_chunks, g, p.reuse_bt);
  int lean_p = -1;  // block position of this thread's box token
  if (p.lean && nrows > 0 && n_in <= p.reuse_chunks * kBN) {
    int r0, nr;
    lean_rows(nrows, split, S, r0, nr);
    if (nr > 0) lr = lean_place(g, row0 + r0, nr);
  }
  const bool lean_early = lr.nr > 0 && p.lean_early;
  if (lr.nr > 0) lean_p = lean_pos(p, q0, lr, tid);
  if (lean_early) lean_issue<kD>(p, ls, s_lean_bar, hk, q0, in0, n_in, lr, tid);
  pdl_wait();
  pdl_trigger();
  // The decision's loads, the state vote's and the early cache rows go out
  // together (the cache rows from warps 1.., after warp 0's decision loads).
  const VoteLoads vote = state_vote_load(p, tid, kThreads);
  DecisionIn din;
  if (tid < g) din = decision_load(p, b, hk * g + tid);
  if (lean_early) lean_fetch<kD>(p, ls, s_lean_bar, hk, in0, n_in, lr, lean_p, tid);
  if (tid < g) s_rec[tid] = decide(p, din) ? 1 : 0;
  const bool need_state = state_vote(vote);
  bool any_rec = false;
  for (int j = 0; j < g; ++j) any_rec |= (s_rec[j] != 0);

  // ------------------------------------------------------------ chunk schedule
  const bool do_out = p.do_out && any_rec;
  const int out_chunks = do_out ? (n_out + kN - 1) / kN : 0;
  const int in_chunks = p.do_in ? (n_in + kN - 1) / kN : 0;
  int pa, pb;
  prefix_range(split, S, out_chunks, in_chunks, pa, pb);
  const bool has_in = p.do_in && split == S - 1;
  const bool has_out = do_out && (pb > pa || (out_chunks == 0 && split == 0));
  const bool cluster_mode = S > 1 && do_out;  // uniform over the cluster
  const bool active = nrows > 0;               // uniform over the cluster
  const int nA = has_in ? in_chunks : 0;       // block chunks, first
  const int nB = has_out ? pb - pa : 0;        // prefix chunks
  const int n_local = nA + nB;
  const bool merger = cluster_mode || has_in || (S == 1 && has_out);

  if (p.decision_out && t == 0 && split == S - 1 && tid < g) p.decision_out[b * p.hq + hk * g + tid] = s_rec[tid];
  // A group whose heads all reuse takes the lean reuse path (its CTAs share the rows).
  const bool lean = p.lean && !any_rec && active;
  if (!lean && lean_early) lean_drain(s_lean_bar, tid);
  if (lean) {
    if (n_in > p.reuse_chunks * kBN) {
      if (tid == 0) record_status(kDevBadIndex);
    } else if (lr.nr > 0) {
      if (!lean_early) {
        lean_issue<kD>(p, ls, s_lean_bar, hk, q0, in0, n_in, lr, tid);
        lean_fetch<kD>(p, ls, s_lean_bar, hk, in0, n_in, lr, lean_p, tid);
      }
      lean_finish<kD>(p, ls, s_lean_bar, lr, q0, hk, n_in, tid, kThreads);
    }
  } else if (active && (has_in || has_out || cluster_mode)) {
    // -------------------------------------------------------- Q rows (before the K/V stream)
    constexpr int kQVec = kM * (kD / 8);
    constexpr int kQPer = (kQVec + kThreads - 1) / kThreads;
    uint4 qv[kQPer];
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * kThreads;
      const int r = v >> 4;
      qv[k] = make_uint4(0u, 0u, 0u, 0u);
      if (v < kQVec && r < nrows) {
        const int rho = row0 + r;
        qv[k] = *reinterpret_cast<const uint4*>(
            p.q + (static_cast<size_t>(q0 + rho / g) * p.hq + hk * g + rho % g) * kD + (v & 15) * 8);
      }
    }
    if (tid < kM) {
      int pos = -1;
      if (tid < nrows) {
        const int rho = row0 + tid;
        pos = p.q_rows ? p.q_rows[q0 + rho / g] : rho / g;
        if (pos < 0 || pos >= n_in) {
          record_status(kDevBadIndex);
          pos = -1;
        } else if (merger && p.fused && !(do_out && s_rec[rho % g])) {
          // cached rows this CTA merges with go to L2 while the attention runs
          const size_t ce = static_cast<size_t>(in0 + pos) * p.hq + hk * g + rho % g;
          prefetch_l2(p.cache_a + ce * kD, kD * 4);
          prefetch_l2_line(p.cache_l + ce);
        }
      }
      s_pos[tid] = pos;
    }

    const uint64_t pol = l2_policy_evict_first();
    auto load = [&](int c, bool is_v) {
      const int st = c % kStages;
      const bool seg_in = c < nA;
      const CUtensorMap* map = is_v ? (seg_in ? &p.tm_v_in : &p.tm_v_out) : (seg_in ? &p.tm_k_in : &p.tm_k_out);
      uint64_t* bar = is_v ? &v_full[st] : &k_full[st];
      uint8_t* dst = smem + (is_v ? kOffV : kOffK) + st * kTile;
      const int y = seg_in ? in0 + c * kN : out0 + (pa + c - nA) * kN;
      mbar_arrive_expect_tx(bar, kTile);
      tma_load_2d(dst, map, bar, hk * kD, y, pol);
      tma_load_2d(dst + kHalf, map, bar, hk * kD + 64, y, pol);
    };
    // The TMA thread initialises the barriers and starts the stream at once.
    if (warp == kTmaWarp && lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&k_full[i], 1);
        mbar_init(&k_empty[i], 1);
        mbar_init(&v_full[i], 1);
        mbar_init(&v_empty[i], 1);
      }
      mbar_init(&s_full[0], 1);
      mbar_init(&s_full[1], 1);
      mbar_init(p_full, kRowThreads * kM / 32);  // one arrival per row warp
      for (int i = 0; i < 4; ++i) {  // two threads per row: the two warps of a lane quarter
        mbar_init(&s_xch[i], 2);   // both values written
        mbar_init(&s_xrd[i], 2);   // both read
      }
      mbar_init(pv_done, 1);
      mbar_init(drain, 1);
      *s_abort = 0;
      fence_barrier_init();
      for (int c = 0; c < min(kStages, n_local); ++c) {
        load(c, false);
        load(c, true);
      }
    }
    if (warp == kMmaWarp && n_local > 0) {
      tmem_alloc(s_tmem, kTmemCols);
      tmem_relinquish();
    }
    // Q tile -> shared memory, 128-byte swizzled K-major (the layout TMA would write)
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * kThreads;
      if (v < kQVec) {
        const int r = v >> 4;
        const int c = v & 15;
        *reinterpret_cast<uint4*>(smem + kOffQ + (c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = qv[k];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    // q_ref follows the queries of heads that recompute (fb_step, block owner)
    if (has_in && p.fused && p.q_ref != nullptr && any_rec) {
#pragma unroll
      for (int k = 0; k < kQPer; ++k) {
        const int v = tid + k * kThreads;
        const int r = v >> 4;
        if (v >= kQVec || r >= nrows) continue;
        const int j = (row0 + r) % g;
        if (!s_rec[j] || s_pos[r] < 0) continue;
        *reinterpret_cast<uint4*>(p.q_ref + (static_cast<size_t>(in0 + s_pos[r]) * p.hq + hk * g + j) * kD +
                                  (v & 15) * 8) = qv[k];
      }
    }

    float m_in = kNegInf, l_in = 0.f, m_out = kNegInf, l_out = 0.f;
    // rows warps only: warp w holds TMEM lanes 32 (w % 4) .. + 31, keys 64 (w / 4) .. + 63
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    if (n_local > 0) {
      if (warp == kTmaWarp) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
          int issued_k = min(kStages, n_local), issued_v = issued_k;
          for (int c = kStages; c < n_local; ++c) {
            if (*s_abort) break;
            const int st = c % kStages;
            const uint32_t ph = (c / kStages - 1) & 1;  // use of the slot by chunk c - kStages
            if (!mbar_wait(&k_empty[st], ph)) {
              record_status(kDevTimeout);
              *s_abort = 1;
              break;
            }
            load(c, false);
            issued_k = c + 1;
            if (!mbar_wait(&v_empty[st], ph)) {
              record_status(kDevTimeout);
              *s_abort = 1;
              break;
            }
            load(c, true);
            issued_v = c + 1;
          }
          if (*s_abort) {  // copies in flight land before the CTA moves on
            for (int c = max(0, issued_k - kStages); c < issued_k; ++c)
              if (!mbar_wait(&k_full[c % kStages], (c / kStages) & 1)) record_status(kDevTimeout);
            for (int c = max(0, issued_v - kStages); c < issued_v; ++c)
              if (!mbar_wait(&v_full[c % kStages], (c / kStages) & 1)) record_status(kDevTimeout);
          }
        }
      } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
          const uint32_t q_a = smem_u32(smem + kOffQ);
          // Descriptors are built once; a K step or a ring slot only moves the
          // start address (16-byte units in the low bits), so the issue loop is a
          // handful of integer adds per MMA.
          const uint64_t dq = sdesc_sw128(q_a, 16, 1024);
          const uint64_t dk = sdesc_sw128(smem_u32(smem + kOffK), 16, 1024);
          const uint64_t dv = sdesc_sw128(smem_u32(smem + kOffV), kHalf, 1024);
          auto issue_s = [&](int c) -> bool {
            const int st = c % kStages;
            if (!mbar_wait(&k_full[st], (c / kStages) & 1)) return false;
            tc_fence_after();
            const uint64_t dks = dk + static_cast<uint64_t>(st * (kTile >> 4));
            const uint32_t d = tmem + kColS + (c & 1) * kN;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
              umma_bf16(d, dq + off, dks + off, kIdescS, kk > 0);
            }
            umma_commit(&s_full[c & 1]);
            umma_commit(&k_empty[st]);
            return true;
          };
          auto issue_pv = [&](int c) -> bool {
            const int st = c % kStages;
            if (!mbar_wait(p_full, c & 1)) return false;
            if (!mbar_wait(&v_full[st], (c / kStages) & 1)) return false;
            tc_fence_after();
            const uint64_t dvs = dv + static_cast<uint64_t>(st * (kTile >> 4));
            const uint32_t pt = tmem + kColS + (c & 1) * kN;  // P(c), packed bf16 pairs
            const bool first = c == 0 || c == nA;
            const uint32_t d = tmem + (c < nA ? kColIn : kColOut);
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk)
              umma_bf16_ts(d, pt + kk * 8, dvs + static_cast<uint64_t>((kk * 16 * 128) >> 4), kIdescO,
                           (first && kk == 0) ? 0u : 1u);
            umma_commit(pv_done);
            umma_commit(&v_empty[st]);
            return true;
          };
          bool ok = true;
          for (int c = 0; c < n_local && ok; ++c) {
            if (*s_abort) {
              ok = false;
              break;
            }
            ok = issue_s(c);
            if (ok && c > 0) ok = issue_pv(c - 1);
          }
          if (ok) ok = issue_pv(n_local - 1);
          if (!ok) {
            record_status(kDevTimeout);
            *s_abort = 1;
          }
          umma_commit(drain);  // every MMA issued has finished before the CTA moves on
          if (!mbar_wait(drain, 0)) record_status(kDevTimeout);
        }
      } else if constexpr (kRowThreads == 2) {
        // ---------------------------------------------------- rows: softmax
        // Two threads per row: warp w takes keys 64 h .. 64 h + 63 (h = w / 4) of
        // the rows of TMEM lane quarter w % 4, so that each SM sub-partition runs
        // two softmax warps that fill each other's stalls.  The halves share the
        // running max of the row (one exchange per chunk) and keep their own sums.
        const int h = warp >> 2;
        const int qr = warp & 3;
        const int r = qr * 32 + lane;  // the row = TMEM lane
        float m = kNegInf, l = 0.f;
        bool ok = true;
        int round = 0;  // exchanges made with the other half's warp
        // this half's value of the row for the other half's, both bounded waits
        auto exchange = [&](float v) -> float {
          if (round > 0 && !__all_sync(0xffffffffu, mbar_wait(&s_xrd[qr], (round - 1) & 1))) ok = false;
          s_xv[h][r] = v;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_xch[qr]);
          if (!__all_sync(0xffffffffu, mbar_wait(&s_xch[qr], round & 1))) ok = false;
          tc_fence_after();
          const float o = s_xv[h ^ 1][r];
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_xrd[qr]);
          ++round;
          return o;
        };
        // skip-mask bits of this half's 64 keys of a prefix chunk, loaded one chunk ahead
        auto skip_of = [&](int c) -> uint64_t {
          if (!p.out_skip || c < nA || c >= n_local) return 0ull;
          return skip_bits64(p.out_skip, p.total_out, out0 + (pa + c - nA) * kN + 64 * h);
        };
        uint64_t skip_next = skip_of(0);
        for (int c = 0; c < n_local; ++c) {
          const uint64_t skip = skip_next;  // bit k: key 64 h + k of the chunk left out
          skip_next = skip_of(c + 1);
          if (c == nA && c > 0) {  // block segment done; the prefix segment starts
            m_in = m;
            l_in = l;
            m = kNegInf;
            l = 0.f;
          }
          const uint32_t sp = lane_base + kColS + (c & 1) * kN;  // S(c), then P(c)
          const bool seg_in = c < nA;
          const int key0 = seg_in ? c * kN : (pa + c - nA) * kN;
          const int valid = min(kN, (seg_in ? n_in : n_out) - key0) - 64 * h;  // of this half's keys
          const bool first = c == 0 || c == nA;
          if (!__all_sync(0xffffffffu, mbar_wait(&s_full[c & 1], (c >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sv[2][32];
          tmem_ld32(sp + 64 * h, sv[0]);
          tmem_ld32(sp + 64 * h + 32, sv[1]);
          tmem_wait_ld();
          reg_fence32(sv[0]);
          reg_fence32(sv[1]);
          // Keys past the segment's end, and prefix keys the skip mask leaves out,
          // get -inf; the row max of the raw scores (the scale is positive, so it
          // commutes with the max) in four chains of 3-input maxima.
          if (valid < 64 || skip) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (32 * i + k >= valid || ((skip >> (32 * i + k)) & 1ull)) sv[i][k] = __float_as_uint(kNegInf);
            }
          }
          float mxa[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int k = 0; k < 32; k += 2)
              mxa[(k >> 1) & 3] = max3(mxa[(k >> 1) & 3], __uint_as_float(sv[i][k]), __uint_as_float(sv[i][k + 1]));
          }
          const float mxh = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
          // Both halves have read their scores once the exchange is through, so P
          // may be written over S below (half 1's P lands on half 0's S columns).
          const float mxo = exchange(mxh);
          if (!ok) break;
          const float mx = fmaxf(mxh, mxo) * p.scale_log2;
          const float m_new = fmaxf(m, mx);
          float alpha = 1.f;
          bool resc = false;
          if (first) {
            m = m_new;
          } else if (m_new > m + kRescaleSlack) {
            alpha = ex2(m - m_new);
            m = m_new;
            resc = true;
          }
          const float nm = m == kNegInf ? 0.f : -m;
          // P = 2^(s * scale - m), rounded to bf16 for the P V product; paired fp32
          // arithmetic, pairs 8a+0..2 of every eight by the cubic, the rest by MUFU;
          // the half-row sum in eight chains (four paired accumulators).
          uint32_t pk[32];  // packed bf16 pairs: keys 64 h + 2j, 64 h + 2j + 1 in column 32 h + j
          uint64_t rsa[4];
#pragma unroll
          for (int a2 = 0; a2 < 4; ++a2) rsa[a2] = 0ull;
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t nm2 = f2_pack(nm, nm);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const uint64_t x = ffma2(f2_pack(__uint_as_float(sv[i][k]), __uint_as_float(sv[i][k + 1])), scale2, nm2);
              float p0, p1;
              if (((k >> 1) & 7) < 3) {
                exp2_poly2(x, p0, p1);
              } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                p0 = ex2(x0);
                p1 = ex2(x1);
              }
              rsa[(k >> 1) & 3] = fadd2(rsa[(k >> 1) & 3], f2_pack(p0, p1));
              pk[16 * i + k / 2] = pack_bf16x2(p0, p1);
            }
          }
          float r0, r1, r2, r3, r4, r5, r6, r7;
          f2_unpack(rsa[0], r0, r1);
          f2_unpack(rsa[1], r2, r3);
          f2_unpack(rsa[2], r4, r5);
          f2_unpack(rsa[3], r6, r7);
          const float rs = ((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7));
          l = l * alpha + rs;
          // P V(c-1) must be finished before O is rescaled; otherwise the wait only
          // keeps the rows in step with the MMA thread (one wait per chunk, before
          // P(c) is published, so the phase waited for is never overtaken).  The
          // decision is the same in both halves (same maxima), each rescales its
          // half of O.
          const bool rescale = __any_sync(0xffffffffu, resc);
          bool waited = c == 0;
          if (rescale) {
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (c - 1) & 1))) {
              ok = false;
              break;
            }
            waited = true;
            tc_fence_after();
            const uint32_t oc = lane_base + (seg_in ? kColIn : kColOut) + 64 * h;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              uint32_t o[32];
              tmem_ld32(oc + 32 * i, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(oc + 32 * i, o);
            }
          }
          // P(c) over S(c) columns whose scores both halves have read (see above)
          tmem_st32(sp + 32 * h, pk);
          tmem_wait_st();
          if (!waited) {
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (c - 1) & 1))) {
              ok = false;
              break;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(pv_done, (n_local - 1) & 1))) ok = false;
        if (!ok) {
          if (lane == 0) record_status(kDevTimeout);
          *s_abort = 1;
        }
        tc_fence_after();
        if (nB > 0) {
          m_out = m;
          l_out = l;
        } else {
          m_in = m;
          l_in = l;
        }
        // the rows' sums: this half's and the other half's
        if (ok) {
          l_in += exchange(l_in);
          l_out += exchange(l_out);
        }
      } else {
        // ---------------------------------------------------- rows: softmax, one thread per row
        float m = kNegInf, l = 0.f;
        bool ok = true;
        // skip-mask bits of a prefix chunk's 128 keys, loaded one chunk ahead
        auto skip_of = [&](int c, uint64_t (&w)[2]) {
          w[0] = w[1] = 0ull;
          if (p.out_skip && c >= nA && c < n_local) {
            const int t0 = out0 + (pa + c - nA) * kN;
            w[0] = skip_bits64(p.out_skip, p.total_out, t0);
            w[1] = skip_bits64(p.out_skip, p.total_out, t0 + 64);
          }
        };
        uint64_t skip_next[2];
        skip_of(0, skip_next);
        for (int c = 0; c < n_local; ++c) {
          const uint64_t skip[2] = {skip_next[0], skip_next[1]};
          skip_of(c + 1, skip_next);
          if (c == nA && c > 0) {  // block segment done; the prefix segment starts
            m_in = m;
            l_in = l;
            m = kNegInf;
            l = 0.f;
          }
          const uint32_t sp = lane_base + kColS + (c & 1) * kN;  // S(c), then P(c)
          const bool seg_in = c < nA;
          const int key0 = seg_in ? c * kN : (pa + c - nA) * kN;
          const int valid = min(kN, (seg_in ? n_in : n_out) - key0);
          const bool first = c == 0 || c == nA;
          if (!__all_sync(0xffffffffu, mbar_wait(&s_full[c & 1], (c >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sv[4][32];
#pragma unroll
          for (int i = 0; i < 4; ++i) tmem_ld32(sp + 32 * i, sv[i]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4; ++i) reg_fence32(sv[i]);
          // Row max of the raw scores (the scale is positive, so it commutes with
          // the max), four independent chains of 3-input maxima.  Keys past the
          // segment's end, and prefix keys the skip mask leaves out, get -inf.
          if (valid < kN || (skip[0] | skip[1])) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (32 * i + k >= valid || ((skip[i >> 1] >> (32 * (i & 1) + k)) & 1ull))
                  sv[i][k] = __float_as_uint(kNegInf);
            }
          }
          float mxa[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int k = 0; k < 32; k += 2)
              mxa[(k >> 1) & 3] = max3(mxa[(k >> 1) & 3], __uint_as_float(sv[i][k]), __uint_as_float(sv[i][k + 1]));
          }
          const float mx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])) * p.scale_log2;
          const float m_new = fmaxf(m, mx);
          float alpha = 1.f;
          bool resc = false;
          if (first) {
            m = m_new;
          } else if (m_new > m + kRescaleSlack) {
            alpha = ex2(m - m_new);
            m = m_new;
            resc = true;
          }
          const float nm = m == kNegInf ? 0.f : -m;
          // P = 2^(s * scale - m), rounded to bf16 for the P V product; paired fp32
          // arithmetic, pairs 8a+0..2 of every eight by the cubic, the rest by MUFU;
          // the row sum in eight chains (four paired accumulators).
          uint32_t pk[2][32];  // packed bf16 pairs: keys 2j, 2j+1 in column j
          uint64_t rsa[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) rsa[a] = 0ull;
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t nm2 = f2_pack(nm, nm);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const uint64_t x = ffma2(f2_pack(__uint_as_float(sv[i][k]), __uint_as_float(sv[i][k + 1])), scale2, nm2);
              float p0, p1;
              if (((k >> 1) & 7) < 3) {
                exp2_poly2(x, p0, p1);
              } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                p0 = ex2(x0);
                p1 = ex2(x1);
              }
              rsa[(k >> 1) & 3] = fadd2(rsa[(k >> 1) & 3], f2_pack(p0, p1));
              pk[i >> 1][(16 * i + k / 2) & 31] = pack_bf16x2(p0, p1);
            }
          }
          float r0, r1, r2, r3, r4, r5, r6, r7;
          f2_unpack(rsa[0], r0, r1);
          f2_unpack(rsa[1], r2, r3);
          f2_unpack(rsa[2], r4, r5);
          f2_unpack(rsa[3], r6, r7);
          const float rs = ((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7));
          l = l * alpha + rs;
          // P V(c-1) must be finished before O is rescaled; otherwise the wait only
          // keeps the rows in step with the MMA thread (one wait per chunk, before
          // P(c) is published, so the phase waited for is never overtaken).
          const bool rescale = __any_sync(0xffffffffu, resc);
          bool waited = c == 0;
          if (rescale) {
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (c - 1) & 1))) {
              ok = false;
              break;
            }
            waited = true;
            tc_fence_after();
            const uint32_t oc = lane_base + (seg_in ? kColIn : kColOut);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t o[32];
              tmem_ld32(oc + 32 * i, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(oc + 32 * i, o);
            }
          }
          // P(c) over the S(c) columns it came from (read above, by this thread)
          tmem_st32(sp, pk[0]);
          tmem_st32(sp + 32, pk[1]);
          tmem_wait_st();
          if (!waited) {
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (c - 1) & 1))) {
              ok = false;
              break;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(pv_done, (n_local - 1) & 1))) ok = false;
        if (!ok) {
          if (lane == 0) record_status(kDevTimeout);
          *s_abort = 1;
        }
        tc_fence_after();
        if (nB > 0) {
          m_out = m;
          l_out = l;
        } else {
          m_in = m;
          l_in = l;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // -------------------------------------------------------- partials -> shared memory
    if (warp < 4 * kRowThreads && n_local > 0) {  // a row's threads: their shares of the columns
      constexpr int kCols = kD / kRowThreads;
      const int r = (warp & 3) * 32 + lane;
      const int h = warp >> 2;
      auto store = [&](float* part, uint32_t col, float mm, float ll) {
        const float inv = ll > 0.f ? 1.f / ll : 0.f;
        float* row = part + r * kPStride + kCols * h;
#pragma unroll
        for (int i = 0; i < kCols / 32; ++i) {
          uint32_t o[32];
          tmem_ld32(lane_base + col + kCols * h + 32 * i, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(row + 32 * i + k) =
                make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                            __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
        }
        if (h == 0) part[kPartL + r] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : kNegInf;
      };
      if (nA > 0) store(part_in, kColIn, m_in, l_in);
      if (nB > 0) store(part_out, kColOut, m_out, l_out);
    }
    tc_fence_before();
    if (cluster_mode) {
      cluster_sync();
    } else {
      __syncthreads();
    }
    if (warp == kMmaWarp && n_local > 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }

    // -------------------------------------------------------- merge
    if (merger) {
      const int rp = cluster_mode ? (nrows + S - 1) / S : nrows;
      const int r_lo = cluster_mode ? split * rp : 0;
      const int r_hi = min(nrows, r_lo + rp);
      const uint32_t out_a = smem_u32(part_out);
      const uint32_t in_a = smem_u32(part_in);
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
      const int n_out_e = cluster_mode ? S : 1;
      const int in_rank = cluster_mode ? S - 1 : 0;
      constexpr int kW0 = kMaxSplits + 1;  // first bookkeeping slot
      float* wt = reinterpret_cast<float*>(smem + kOffQ);  // the Q tile is dead by now
      // Phase W, one thread per row: the weights of every partial of the row.
      for (int r = r_lo + tid; r < r_hi; r += kThreads) {
        float* wr = wt + (r - r_lo) * kWt;
        const int pos = s_pos[r];
        const int rho = row0 + r;
        const int j = rho % g;
        float kind = 0.f;
        float lo2 = kNegInf, li2 = kNegInf;
        wr[kMaxSplits] = 0.f;
        if (pos >= 0) {
          const int ce = (in0 + pos) * p.hq + hk * g + j;
          wr[kW0 + 4] = __int_as_float(ce);
          wr[kW0 + 5] = __int_as_float((q0 + rho / g) * p.hq + hk * g + j);
          if (do_out && s_rec[j]) {
            float l2[kMaxSplits];
#pragma unroll
            for (int k = 0; k < kMaxSplits; ++k) {
              l2[k] = kNegInf;
              if (k < n_out_e && ((owners >> k) & 1u)) l2[k] = ld_f(out_a, k, kPartL + r) * kLog2e;
            }
            lo2 = log2_weights<kMaxSplits>(l2, wr);
            kind = 1.f;
          } else if (p.fused) {
            lo2 = p.cache_l[ce] * kLog2e;
            kind = 2.f;
          } else {
            kind = 3.f;  // block pass alone
          }
          if (p.do_in) {
            li2 = ld_f(in_a, in_rank, kPartL + r) * kLog2e;
            wr[kMaxSplits] = li2 == kNegInf ? 0.f : 1.f;
          }
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
          wr[kMaxSplits] *= wi;
        }
        wr[kW0 + 0] = wo;
        wr[kW0 + 1] = lo2 == kNegInf ? kNegInf : lo2 * kLn2;
        wr[kW0 + 2] = lf2 == kNegInf ? kNegInf : lf2 * kLn2;
        wr[kW0 + 3] = kind;
      }
      __syncthreads();
      // Phase C, (row, 4 columns) items: loads and multiply-adds only.  Items go
      // in batches of kU per thread, all of a batch's loads issued before any of
      // its stores, so several cache and partial loads are in flight at once.
      constexpr int kC4 = kD / 4;
      constexpr int kU = 8;
      const int n_items = (r_hi - r_lo) * kC4;
      for (int base = tid; base < n_items; base += kThreads * kU) {
        float4 ao[kU], ai[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int item = base + u * kThreads;
          ao[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          ai[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (item >= n_items) continue;
          const int r = r_lo + item / kC4;
          const int c4 = (item % kC4) * 4;
          const float* wr = wt + (r - r_lo) * kWt;
          const int kind = static_cast<int>(wr[kW0 + 3]);
          if (kind == 2) {
            const size_t ce = static_cast<unsigned>(__float_as_int(wr[kW0 + 4]));
            ao[u] = *reinterpret_cast<const float4*>(p.cache_a + ce * kD + c4);
          } else if (kind == 1) {  // the prefix partials of the row, combined here (before any store)
#pragma unroll
            for (int k = 0; k < kMaxSplits; ++k)
              if (wr[k] != 0.f) fma4(ao[u], wr[k], ld_f4(out_a, k, r * kPStride + c4));
          }
          if (kind != 0 && p.do_in && wr[kMaxSplits] != 0.f) ai[u] = ld_f4(in_a, in_rank, r * kPStride + c4);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int item = base + u * kThreads;
          if (item >= n_items) continue;
          const int r = r_lo + item / kC4;
          const int c4 = (item % kC4) * 4;
          const float* wr = wt + (r - r_lo) * kWt;
          const int kind = static_cast<int>(wr[kW0 + 3]);
          if (kind == 0) continue;
          const size_t ce = static_cast<unsigned>(__float_as_int(wr[kW0 + 4]));
          const size_t fe = static_cast<unsigned>(__float_as_int(wr[kW0 + 5]));
          if (kind == 1) {
            *reinterpret_cast<float4*>(p.cache_a + ce * kD + c4) = ao[u];
            if (c4 == 0) p.cache_l[ce] = wr[kW0 + 1];
          }
          if (!p.do_in) continue;
          float4 a_i = make_float4(0.f, 0.f, 0.f, 0.f);
          fma4(a_i, wr[kMaxSplits], ai[u]);
          if (!p.fused) {
            *reinterpret_cast<float4*>(p.a_in + fe * kD + c4) = a_i;
            if (c4 == 0) p.l_in[fe] = wr[kW0 + 2];
            continue;
          }
          const float wo = wr[kW0 + 0];
          const float4 a_o = ao[u];
          __nv_bfloat16* dst = p.a_full + fe * kD + c4;
          *reinterpret_cast<__nv_bfloat162*>(dst) =
              __floats2bfloat162_rn(fmaf(wo, a_o.x, a_i.x), fmaf(wo, a_o.y, a_i.y));
          *reinterpret_cast<__nv_bfloat162*>(dst + 2) =
              __floats2bfloat162_rn(fmaf(wo, a_o.z, a_i.z), fmaf(wo, a_o.w, a_i.w));
          if (c4 == 0 && p.l_full) p.l_full[fe] = wr[kW0 + 2];
        }
      }
    }
    if (cluster_mode) cluster_sync();  // no CTA leaves while its partials may still be read
  }

  // ------------------------------------------------------------ cache-state epilogue
  if (need_state) state_epilogue(p, tid, kThreads, &s_flag);
}

}  // namespace fb
