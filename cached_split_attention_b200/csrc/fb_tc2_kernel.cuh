// Two-tile ("ping-pong") tensor-core kernel for the fused step of multi-head
// attention with large blocks (head_dim 128, one q-head per kv-head, at least
// two 128-row tiles per head): the video-shaped block of 1560 tokens.
//
// A CTA owns 256 rows of one (sequence, head): tile A (rows 0-127) and tile B
// (rows 128-255).  Both tiles share every K/V chunk of 128 keys, so each byte
// brought into shared memory feeds twice the tensor work of the single-tile
// kernel, and the tensor core alternates between the tiles:
//
//     S_A(c)  S_B(c)  PV_A(c)  S_A(c+1)  PV_B(c)  S_B(c+1)  PV_A(c+1) ...
//
// while softmax A works on S_A(c) the tensor core runs PV_B(c-1) and S_B(c), and
// the other way round.  The two softmaxes run concurrently, one warp of each per
// SM sub-partition: a single softmax warp is bound by its own latencies (TMEM
// loads, the exponentials), and the other tile's warp fills its stalls.  (Making
// them take turns, so that each ran alone while the tensor core worked on the
// other tile, measured slower: 460 against 442 us for the video block's
// all-recompute call.)  Warps 0-3 are tile A's rows, warps 4-7 tile B's (thread =
// row = TMEM lane), warp 8 streams K/V with TMA, warp 9 issues the MMAs.
//
// One accumulator per tile.  A head that recomputes streams its prefix chunks
// first; at the boundary the accumulator holds the prefix partial, which is
// normalised and written to the cache as (A_out, L_out) (FlashBlock, "Mecanismo
// Central": the cached out-of-block output); the block chunks then continue the
// same online softmax, so the final accumulator is attention over J_out and J_in,
// which is what the log-space merge of the two partials computes.  A head that
// reuses streams only its block chunks and merges the result with the cached
// partial row by row.
//
// TMEM (512 columns): S_A / P_A at 0, S_B / P_B at 128, O_A at 256, O_B at 384.
// P(c) overwrites S(c) in place; S(c+1) of the same tile is issued after PV(c)
// and the tensor core runs MMAs in issue order, so the completion of S(c+1)
// (its mbarrier) also tells the rows that PV(c) is done and O may be rescaled.
#pragma once

#include "fb_tc_kernel.cuh"

namespace fb {
namespace tc2 {

constexpr int kD = 128;
constexpr int kM = 128;  // rows per tile
constexpr int kN = 128;  // keys per chunk
constexpr int kThreads = 320;
constexpr int kHalf = kN * 128;
constexpr int kTile = 2 * kHalf;  // 32 KB
constexpr int kStages = 2;
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kStages * kTile;
constexpr int kOffQ = kOffV + kStages * kTile;  // Q_A, then Q_B
constexpr int kOffBar = kOffQ + 2 * kTile;
constexpr int kNumBars = 16;
constexpr int kOffPos = kOffBar + kNumBars * 8;
constexpr int kOffMisc = kOffPos + 2 * kM * 4;
constexpr int kSmem = 1024 + kOffMisc + 16;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescS = idesc_bf16(kM, kN, false);
constexpr uint32_t kIdescO = idesc_bf16(kM, kD, true);

static_assert(kSmem <= 232448, "shared memory per CTA");

}  // namespace tc2

__global__ void __launch_bounds__(tc2::kThreads, 1) tc2_attn_kernel(const __grid_constant__ Params p) {
  prefetch_maps(p);
  pdl_wait();
  pdl_trigger();
  using namespace tc2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* k_full = bars;        // [2] TMA -> MMA
  uint64_t* k_empty = bars + 2;   // [2] MMA -> TMA
  uint64_t* v_full = bars + 4;    // [2]
  uint64_t* v_empty = bars + 6;   // [2]
  uint64_t* s_full = bars + 8;    // [tile] MMA -> rows
  uint64_t* p_full = bars + 10;   // [tile] rows -> MMA
  uint64_t* o_done = bars + 12;   // [tile] MMA -> rows, after the last PV
  uint64_t* drain = bars + 14;    // MMA -> MMA
  int* s_pos = reinterpret_cast<int*>(smem + kOffPos);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  __shared__ int s_flag;
  __shared__ int s_rec0;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int item = p.order ? p.order[blockIdx.x] : static_cast<int>(blockIdx.x);  // (b, h, pair)
  const int pair = item % p.tiles;  // p.tiles counts 256-row pairs here
  const int h = item / p.tiles % p.hq;
  const int b = item / p.tiles / p.hq;

  // ------------------------------------------------------------ metadata
  const int q0 = p.cu_q[b];
  const int n_q = p.cu_q[b + 1] - q0;
  const int out0 = p.cu_out[b];
  const int n_out = p.cu_out[b + 1] - out0;
  const int in0 = p.cu_in[b];
  const int n_in = p.cu_in[b + 1] - in0;
  const VoteLoads vote = state_vote_load(p, tid, kThreads);
  if (tid == 0) s_rec0 = head_recompute(p, b, h) ? 1 : 0;
  const bool need_state = state_vote(vote);
  const bool rec = s_rec0 != 0;
  const bool ranges_ok = q0 >= 0 && n_q >= 0 && q0 + n_q <= p.total_q && out0 >= 0 && n_out >= 0 &&
                         out0 + n_out <= p.total_out && in0 >= 0 && n_in >= 0 && in0 + n_in <= p.total_in &&
                         n_q <= n_in;
  const int row0 = pair * 2 * kM;
  if (!ranges_ok && tid == 0 && pair == 0) record_status(kDevBadIndex);
  const int nrows = ranges_ok ? max(0, min(2 * kM, n_q - row0)) : 0;
  if (p.decision_out && pair == 0 && tid == 0) p.decision_out[b * p.hq + h] = rec ? 1 : 0;

  const int nB = rec ? (n_out + kN - 1) / kN : 0;  // prefix chunks, first
  const int nA = (n_in + kN - 1) / kN;             // block chunks
  const int n_chunks = nB + nA;

  if (nrows > 0) {
    // -------------------------------------------------------- Q rows (before the K/V stream)
    constexpr int kQVec = 2 * kM * (kD / 8);
    constexpr int kQPer = (kQVec + kThreads - 1) / kThreads;
    uint4 qv[kQPer];
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * kThreads;
      const int r = v >> 4;
      qv[k] = make_uint4(0u, 0u, 0u, 0u);
      if (v < kQVec && r < nrows)
        qv[k] = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(q0 + row0 + r) * p.hq + h) * kD +
                                                (v & 15) * 8);
    }
    if (tid < 2 * kM) {
      int pos = -1;
      if (tid < nrows) {
        pos = p.q_rows ? p.q_rows[q0 + row0 + tid] : row0 + tid;
        if (pos < 0 || pos >= n_in) {
          record_status(kDevBadIndex);
          pos = -1;
        } else if (!rec) {
          const size_t ce = static_cast<size_t>(in0 + pos) * p.hq + h;
          prefetch_l2(p.cache_a + ce * kD, kD * 4);
          prefetch_l2_line(p.cache_l + ce);
        }
      }
      s_pos[tid] = pos;
    }

    const uint64_t pol = l2_policy_evict_first();
    auto load = [&](int c, bool is_v) {
      const int st = c % kStages;
      const bool seg_out = c < nB;
      const CUtensorMap* map = is_v ? (seg_out ? &p.tm_v_out : &p.tm_v_in) : (seg_out ? &p.tm_k_out : &p.tm_k_in);
      uint64_t* bar = is_v ? &v_full[st] : &k_full[st];
      uint8_t* dst = smem + (is_v ? kOffV : kOffK) + st * kTile;
      const int y = seg_out ? out0 + c * kN : in0 + (c - nB) * kN;
      mbar_arrive_expect_tx(bar, kTile);
      tma_load_2d(dst, map, bar, h * kD, y, pol);
      tma_load_2d(dst + kHalf, map, bar, h * kD + 64, y, pol);
    };
    if (warp == 8 && lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&k_full[i], 1);
        mbar_init(&k_empty[i], 1);
        mbar_init(&v_full[i], 1);
        mbar_init(&v_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&s_full[i], 1);
        mbar_init(&p_full[i], kM / 32);  // one arrival per row warp of the tile
        mbar_init(&o_done[i], 1);
      }
      mbar_init(drain, 1);
      *s_abort = 0;
      fence_barrier_init();
      for (int c = 0; c < min(kStages, n_chunks); ++c) {
        load(c, false);
        load(c, true);
      }
    }
    if (warp == 9) {
      tmem_alloc(s_tmem, kTmemCols);
      tmem_relinquish();
    }
    // Q tiles -> shared memory, 128-byte swizzled K-major
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int v = tid + k * kThreads;
      if (v < kQVec) {
        const int r = v >> 4;
        const int c = v & 15;
        *reinterpret_cast<uint4*>(smem + kOffQ + (r >> 7) * kTile + (c >> 3) * kHalf + (r & 127) * 128 +
                                  (((c & 7) ^ (r & 7)) << 4)) = qv[k];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    if (rec && p.q_ref != nullptr) {  // q_ref follows the queries of a head that recomputes
#pragma unroll
      for (int k = 0; k < kQPer; ++k) {
        const int v = tid + k * kThreads;
        const int r = v >> 4;
        if (v >= kQVec || r >= nrows || s_pos[r] < 0) continue;
        *reinterpret_cast<uint4*>(p.q_ref + (static_cast<size_t>(in0 + s_pos[r]) * p.hq + h) * kD + (v & 15) * 8) =
            qv[k];
      }
    }

    if (warp == 8) {
      // ---------------------------------------------------- TMA producer
      if (lane == 0) {
        int issued_k = min(kStages, n_chunks), issued_v = issued_k;
        for (int c = kStages; c < n_chunks; ++c) {
          if (*s_abort) break;
          const int st = c % kStages;
          const uint32_t ph = (c / kStages - 1) & 1;
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
        if (*s_abort) {
          for (int c = max(0, issued_k - kStages); c < issued_k; ++c)
            if (!mbar_wait(&k_full[c % kStages], (c / kStages) & 1)) record_status(kDevTimeout);
          for (int c = max(0, issued_v - kStages); c < issued_v; ++c)
            if (!mbar_wait(&v_full[c % kStages], (c / kStages) & 1)) record_status(kDevTimeout);
        }
      }
    } else if (warp == 9) {
      // ---------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint64_t dq = sdesc_sw128(smem_u32(smem + kOffQ), 16, 1024);
        const uint64_t dk = sdesc_sw128(smem_u32(smem + kOffK), 16, 1024);
        const uint64_t dv = sdesc_sw128(smem_u32(smem + kOffV), kHalf, 1024);
        auto issue_s = [&](int x, int c) -> bool {
          const int st = c % kStages;
          if (x == 0) {
            if (!mbar_wait(&k_full[st], (c / kStages) & 1)) return false;
            tc_fence_after();
          }
          const uint64_t dqx = dq + static_cast<uint64_t>(x * (kTile >> 4));
          const uint64_t dks = dk + static_cast<uint64_t>(st * (kTile >> 4));
          const uint32_t d = tmem + x * kN;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
            umma_bf16(d, dqx + off, dks + off, kIdescS, kk > 0);
          }
          umma_commit(&s_full[x]);
          if (x == 1) umma_commit(&k_empty[st]);
          return true;
        };
        auto issue_pv = [&](int x, int c) -> bool {
          const int st = c % kStages;
          if (!mbar_wait(&p_full[x], c & 1)) return false;
          if (x == 0 && !mbar_wait(&v_full[st], (c / kStages) & 1)) return false;
          tc_fence_after();
          const uint64_t dvs = dv + static_cast<uint64_t>(st * (kTile >> 4));
          const uint32_t pt = tmem + x * kN;
          const uint32_t d = tmem + 256 + x * kD;
#pragma unroll
          for (int kk = 0; kk < kN / 16; ++kk)
            umma_bf16_ts(d, pt + kk * 8, dvs + static_cast<uint64_t>((kk * 16 * 128) >> 4), kIdescO,
                         (c == 0 && kk == 0) ? 0u : 1u);
          if (c == n_chunks - 1) umma_commit(&o_done[x]);
          if (x == 1) umma_commit(&v_empty[st]);
          return true;
        };
        bool ok = issue_s(0, 0) && issue_s(1, 0);
        for (int c = 0; c < n_chunks && ok; ++c) {
          if (*s_abort) {
            ok = false;
            break;
          }
          ok = issue_pv(0, c);
          if (ok && c + 1 < n_chunks) ok = issue_s(0, c + 1);
          if (ok) ok = issue_pv(1, c);
          if (ok && c + 1 < n_chunks) ok = issue_s(1, c + 1);
        }
        if (!ok) {
          record_status(kDevTimeout);
          *s_abort = 1;
        }
        umma_commit(drain);
        if (!mbar_wait(drain, 0)) record_status(kDevTimeout);
      }
    } else {
      // ---------------------------------------------------- rows: softmax of one tile
      const int x = warp >> 2;            // tile
      const int r = tid & 127;            // row in the tile = TMEM lane
      const int rr = x * kM + r;          // row in the CTA
      const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t sp = lane_base + x * kN;         // S_x, then P_x
      const uint32_t op = lane_base + 256 + x * kD;   // O_x
      const int pos = s_pos[rr];
      const bool row_ok = rr < nrows && pos >= 0;
      const size_t ce = static_cast<size_t>(in0 + max(pos, 0)) * p.hq + h;
      const size_t fe = static_cast<size_t>(q0 + row0 + rr) * p.hq + h;
      float m = kNegInf, l = 0.f;
      bool ok = true;
      const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
      // (A_out, L_out) of the accumulator so far -> cache (prefix partial)
      auto snapshot = [&]() {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t o[32];
          if (nB > 0) {
            tmem_ld32(op + 32 * i, o);
            tmem_wait_ld();
            reg_fence32(o);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0u;
          }
          if (row_ok) {
            float* dst = p.cache_a + ce * kD + 32 * i;
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(dst + k) =
                  make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                              __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
          }
        }
        if (row_ok) p.cache_l[ce] = l > 0.f ? (m + log2f(l)) * kLn2 : kNegInf;
      };
      if (rec && nB == 0) snapshot();  // empty prefix: (0, -inf)
      // skip-mask bits of a prefix chunk's 128 keys, loaded one chunk ahead
      auto skip_of = [&](int c, uint64_t (&w)[2]) {
        w[0] = w[1] = 0ull;
        if (p.out_skip && c < nB) {
          w[0] = skip_bits64(p.out_skip, p.total_out, out0 + c * kN);
          w[1] = skip_bits64(p.out_skip, p.total_out, out0 + c * kN + 64);
        }
      };
      uint64_t skip_next[2];
      skip_of(0, skip_next);
      for (int c = 0; c < n_chunks; ++c) {
        const bool seg_out = c < nB;
        const int key0 = seg_out ? c * kN : (c - nB) * kN;
        const int valid = min(kN, (seg_out ? n_out : n_in) - key0);
        const uint64_t skip[2] = {skip_next[0], skip_next[1]};  // bit k: key key0 + k (+ 64) left out
        skip_of(c + 1, skip_next);
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[x], c & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();  // S(c) done, and with it every earlier MMA (PV(c-1) included)
        if (rec && c == nB && nB > 0) snapshot();
        // row max of the raw scores (the whole S row in one TMEM round trip); the
        // first 64 columns stay in registers for the exponentials
        float mxa[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
        uint32_t sk[2][32];
        {
          uint32_t sv[2][32];
          tmem_ld32(sp, sk[0]);
          tmem_ld32(sp + 32, sk[1]);
          tmem_ld32(sp + 64, sv[0]);
          tmem_ld32(sp + 96, sv[1]);
          tmem_wait_ld();
          reg_fence32(sk[0]);
          reg_fence32(sk[1]);
          reg_fence32(sv[0]);
          reg_fence32(sv[1]);
          if (valid < kN || (skip[0] | skip[1])) {  // ragged last chunk of a segment, skipped keys
#pragma unroll
            for (int i = 0; i < 2; ++i) {
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                if (32 * i + k >= valid || ((skip[0] >> (32 * i + k)) & 1ull)) sk[i][k] = __float_as_uint(kNegInf);
                if (64 + 32 * i + k >= valid || ((skip[1] >> (32 * i + k)) & 1ull))
                  sv[i][k] = __float_as_uint(kNegInf);
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              mxa[(k >> 1) & 3] =
                  tc::max3(mxa[(k >> 1) & 3], __uint_as_float(sk[i][k]), __uint_as_float(sk[i][k + 1]));
              mxa[(k >> 1) & 3] =
                  tc::max3(mxa[(k >> 1) & 3], __uint_as_float(sv[i][k]), __uint_as_float(sv[i][k + 1]));
            }
          }
        }
        const float mx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])) * p.scale_log2;
        const float m_new = fmaxf(m, mx);
        float alpha = 1.f;
        bool resc = false;
        if (c == 0) {
          m = m_new;
        } else if (m_new > m + tc::kRescaleSlack) {
          alpha = ex2(m - m_new);
          m = m_new;
          resc = true;
        }
        if (__any_sync(0xffffffffu, resc)) {  // PV(c-1) is done (see above)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t o[32];
            tmem_ld32(op + 32 * i, o);
            tmem_wait_ld();
            reg_fence32(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(op + 32 * i, o);
          }
        }
        const uint64_t nm2 = f2_pack(m == kNegInf ? 0.f : -m, m == kNegInf ? 0.f : -m);
        // P = 2^(s * scale - m): the kept first half while the second half comes
        // back from TMEM; each 32-column group of P is stored over S columns whose
        // scores are already in registers
        uint64_t rsa[2] = {0ull, 0ull};
        auto exp_group = [&](const uint32_t (&sg)[32], uint32_t col) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const uint64_t xx = ffma2(f2_pack(__uint_as_float(sg[k]), __uint_as_float(sg[k + 1])), scale2, nm2);
            float p0, p1;
            if (((k >> 1) & 7) < 3) {
              tc::exp2_poly2(xx, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(xx, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            rsa[(k >> 1) & 1] = fadd2(rsa[(k >> 1) & 1], f2_pack(p0, p1));
            pk[k >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st16(sp + col, pk);
        };
        uint32_t sh[2][32];
        tmem_ld32(sp + 64, sh[0]);
        tmem_ld32(sp + 96, sh[1]);
        exp_group(sk[0], 0);
        exp_group(sk[1], 16);
        tmem_wait_ld();
        reg_fence32(sh[0]);
        reg_fence32(sh[1]);
        if (valid < kN || skip[1]) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (64 + 32 * i + k >= valid || ((skip[1] >> (32 * i + k)) & 1ull)) sh[i][k] = __float_as_uint(kNegInf);
          }
        }
        exp_group(sh[0], 32);
        exp_group(sh[1], 48);
        float r0, r1, r2, r3;
        f2_unpack(rsa[0], r0, r1);
        f2_unpack(rsa[1], r2, r3);
        l = l * alpha + ((r0 + r1) + (r2 + r3));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&o_done[x], 0))) ok = false;
      if (!ok) {
        if (lane == 0) record_status(kDevTimeout);
        *s_abort = 1;
      }
      tc_fence_after();
      // -------------------------------------------------- epilogue, one row per thread
      // rec: the accumulator is attention over J_out and J_in (the merge, exact);
      // reuse: the block partial, merged here with the cached prefix partial.
      float lo = kNegInf, li = l > 0.f ? m + log2f(l) : kNegInf;  // base 2
      float wo = 0.f, wi = 1.f;
      if (!rec && row_ok) {
        lo = p.cache_l[ce] * kLog2e;
        const float m2 = fmaxf(lo, li);
        if (m2 == kNegInf) {
          wi = 0.f;
        } else {
          wo = lo == kNegInf ? 0.f : ex2(lo - m2);
          wi = li == kNegInf ? 0.f : ex2(li - m2);
          const float inv = rcp_approx(wo + wi);
          li = m2 + lg2_approx(wo + wi);
          wo *= inv;
          wi *= inv;
        }
      }
      const float inv_l = l > 0.f ? wi / l : 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t o[32];
        tmem_ld32(op + 32 * i, o);
        tmem_wait_ld();
        reg_fence32(o);
        if (!row_ok) continue;
        const float* co = p.cache_a + ce * kD + 32 * i;
        __nv_bfloat16* dst = p.a_full + fe * kD + 32 * i;
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
          float a[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(o[k + e]) * inv_l;
          if (!rec) {
            const float4 c0 = *reinterpret_cast<const float4*>(co + k);
            const float4 c1 = *reinterpret_cast<const float4*>(co + k + 4);
            a[0] = fmaf(wo, c0.x, a[0]);
            a[1] = fmaf(wo, c0.y, a[1]);
            a[2] = fmaf(wo, c0.z, a[2]);
            a[3] = fmaf(wo, c0.w, a[3]);
            a[4] = fmaf(wo, c1.x, a[4]);
            a[5] = fmaf(wo, c1.y, a[5]);
            a[6] = fmaf(wo, c1.z, a[6]);
            a[7] = fmaf(wo, c1.w, a[7]);
          }
          *reinterpret_cast<uint4*>(dst + k) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                                          pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        }
      }
      if (row_ok && p.l_full) p.l_full[fe] = li == kNegInf ? kNegInf : li * kLn2;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  }

  // ------------------------------------------------------------ cache-state epilogue
  if (need_state) state_epilogue(p, tid, kThreads, &s_flag);
}

}  // namespace fb
