// Lean reuse path of the fused FlashBlock step (sm_100a).
//
// On a reuse step the out-of-block partial (A_out, L_out) comes from the cache, so
// the only attention left is the block's own: every active query row against the
// block's B keys (bidirectional), followed by the log-space merge with the cached
// row (FlashBlock, "Mecanismo Central": the stored values are reused instead of
// reading the prefix K/V again).  That is a few MB per call and a short chain of
// dependent loads, so when no head of a group (sequence, kv-head, row tile)
// recomputes, the streaming kernels hand the group to this path instead of their
// TMA pipeline, cluster and merge phases.  The group's CTAs share its rows (whole
// 16-row warp slabs); each CTA
//
//   loads      by TMA on one mbarrier: the block K/V of the kv-head as 64-row
//              boxes (whole 64-key chunks; keys past the block are masked) and its
//              Q rows as one {64 columns, g heads, bt tokens} box per 64 columns,
//              both in the 128-byte swizzled layout; and on a second mbarrier each
//              token's g cached A_out rows as one 1-D bulk copy (one expect-tx for
//              the CTA), its L_out entries by cp.async;
//   attends    S = Q K^T and O = P V with mma.sync (bf16 in, fp32 accumulate),
//              online softmax in base 2 (the streaming kernel's inner loop);
//   merges     in registers: A_full = w_out A_out + w_in A_in, L_full =
//              logaddexp(L_out, L_in), written as bf16 / fp32.
//
// When the grid fits in one wave (`lean_early`), the loads do not wait for the
// reuse decision: the block inputs and the index arrays go out before the wait
// for the previous kernel of the stream (no kernel that lets this one start early
// writes them), the cached rows right after it, beside the decision's own loads;
// a CTA whose group recomputes after all lets the copies land before the
// streaming path reuses the shared memory.  Otherwise a CTA loads only once it knows its group
// reuses.  Blocks of up to kMaxKeys keys take this path (the host plan checks
// max_kv_in and the shared memory it needs); longer blocks are real contractions
// and stay on the streaming pipelines.
//
// Included by fb_kernels.cuh after the helpers it shares with the warp-MMA kernel
// (Params, Acc, consume_keys) and before the kernels that call it.
#pragma once

namespace fb {
namespace reuse {

constexpr int kMaxKeys = 128;  // block keys a CTA holds: two 64-key chunks

__host__ __device__ constexpr int tile_bytes(int d) { return kBN * d * 2; }
// Tokens of a CTA's Q box: any `nr_max` consecutive rows, starting anywhere inside
// a token of g rows, lie in this many tokens (and so do the slabs' padding rows).
__host__ __device__ constexpr int box_tokens(int g, int nr_max) { return (nr_max + 2 * g - 2) / g; }
// Rows of a 64-column Q half in shared memory (a whole number of 8-row swizzle atoms).
__host__ __device__ constexpr int box_rows(int g, int bt) { return (g * bt + 7) / 8 * 8; }
__host__ __device__ constexpr int align16(int x) { return (x + 15) / 16 * 16; }
// Shared memory of the lean path for `chunks` 64-key chunks and a Q box of bt
// tokens x g heads, after the 1024-byte alignment of the kernel's base: K, V
// chunks; Q halves; cached A rows (fp32, unpadded); cached L; each token's position.
__host__ __device__ constexpr int smem_bytes(int d, int chunks, int g, int bt) {
  return 2 * chunks * tile_bytes(d) + (d / 64) * box_rows(g, bt) * 128 + g * bt * d * 4 + align16(g * bt * 4) +
         align16(bt * 4);
}

}  // namespace reuse

// Where a lean CTA's rows [rho0, rho0 + nr) of its sequence (row rho = token
// rho / g, head rho % g of the kv-head) sit in its box: tokens tok_lo ..
// tok_lo + ntok - 1, row rho at box row rho - tok_lo * g, the first at `off`.
struct LeanRows {
  int rho0, nr, tok_lo, ntok, off;
};

__device__ __forceinline__ LeanRows lean_place(int g, int rho0, int nr) {
  LeanRows lr;
  lr.rho0 = rho0;
  lr.nr = nr;
  lr.tok_lo = rho0 / g;
  lr.ntok = (rho0 + nr - 1) / g - lr.tok_lo + 1;
  lr.off = rho0 - lr.tok_lo * g;
  return lr;
}

// The lean path's regions of the kernel's 1024-byte aligned dynamic shared memory.
template <int D>
struct LeanSmem {
  uint8_t* ks;  // K chunks, 64 keys each, two 64-column halves per chunk
  uint8_t* vs;  // V chunks
  uint8_t* qs;  // Q halves, box_rows(g, bt) rows of 128 bytes each
  float* ca;    // cached A_out, box row R at ca + R * D
  float* cl;    // cached L_out of box row R
  int* pos;     // block position of box token t (-1: out of range)
  int qrows;
  __device__ __forceinline__ LeanSmem(uint8_t* smem, int nch, int g, int bt) {
    constexpr int kT = reuse::tile_bytes(D);
    qrows = reuse::box_rows(g, bt);
    ks = smem;
    vs = smem + nch * kT;
    qs = smem + 2 * nch * kT;
    ca = reinterpret_cast<float*>(qs + (D / 64) * qrows * 128);
    cl = ca + g * bt * D;
    pos = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(cl) + reuse::align16(g * bt * 4));
  }
};

// The rows of a served group that CTA `split` of its S takes: whole 16-row warp
// slabs, dealt out as evenly as the slabs allow.
__device__ __forceinline__ void lean_rows(int nrows, int split, int S, int& r0, int& nr) {
  const int slabs = (nrows + 15) / 16;
  const int per = (slabs + S - 1) / S;
  r0 = min(nrows, split * per * 16);
  nr = min(nrows, (split + 1) * per * 16) - r0;
}

// Box token t has a thread of warps 1.. (warp 0 is left to the reuse decision's
// loads), dealt round-robin over those warps so that each issues few of the
// per-token copies (a warp issues its lanes' bulk copies one after another): token
// t = lane * W + (warp - 1) with W = warps - 1.  The host plan keeps bt <= 32 W.
constexpr int kLeanTok0 = 32;
__device__ __forceinline__ int lean_tok(int tid) {
  const int w1 = static_cast<int>(blockDim.x >> 5) - 1;
  const int w = (tid >> 5) - 1;
  return w < 0 ? -1 : (tid & 31) * w1 + w;
}

// Block position of the box token of thread `tid` (-1: none).  Read from q_rows
// before the dependency wait; the caller has checked the sequence's ranges.
__device__ __forceinline__ int lean_pos(const Params& p, int q0, const LeanRows& lr, int tid) {
  const int t = lean_tok(tid);
  if (t < 0 || t >= lr.ntok) return -1;
  const int tok = lr.tok_lo + t;
  return p.q_rows ? p.q_rows[q0 + tok] : tok;
}

// Before the dependency wait: thread 0 arms the two barriers (0: block K/V and Q;
// 1: the cached rows) and issues the K/V chunks and the Q box.  Every thread of the
// CTA calls it (it has a CTA barrier).
template <int D>
__device__ __forceinline__ void lean_issue(const Params& p, const LeanSmem<D>& ls, uint64_t* bars, int hk, int q0,
                                           int in0, int n_in, const LeanRows& lr, int tid) {
  constexpr int kT = reuse::tile_bytes(D);
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    const int used = (n_in + kBN - 1) / kBN;  // 64-key chunks holding the block
    // a box counts in full, zero-filled rows past the tensor's end included
    mbar_arrive_expect_tx(&bars[0], 2 * used * kT + (D / 64) * p.g * p.reuse_bt * 128);
    for (int c = 0; c < used; ++c) {
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_2d_plain(ls.ks + c * kT + hh * (kBN * 128), &p.tm_k_lean, &bars[0], hk * D + hh * 64, in0 + c * kBN);
        tma_load_2d_plain(ls.vs + c * kT + hh * (kBN * 128), &p.tm_v_lean, &bars[0], hk * D + hh * 64, in0 + c * kBN);
      }
    }
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh)
      tma_load_3d_plain(ls.qs + hh * ls.qrows * 128, &p.tm_q_lean, &bars[0], hh * 64, hk * p.g, q0 + lr.tok_lo);
  }
}

// Every thread waits for the block K/V and Q; on a timeout (never expected) the
// copies still in flight get a second bounded wait.  False: the inputs may be
// incomplete (the status is recorded and the CTA writes nothing).
__device__ __forceinline__ bool lean_wait(uint64_t* bar, int tid) {
  if (mbar_wait(bar, 0)) return true;
  if (tid == 0) record_status(kDevTimeout);
  mbar_wait(bar, 0);
  return false;
}

// Block attention of warp slab `slab` (box rows off + 16 slab ..): the running
// state of its 16 rows, unnormalised, in `acc`.
template <int D>
__device__ __forceinline__ void lean_attend(const Params& p, const LeanSmem<D>& ls, const LeanRows& lr, int slab,
                                            int lane, int n_in, Acc<D>& acc) {
  constexpr int kT = reuse::tile_bytes(D);
  uint32_t qf[D / 16][4];
  const int R = lr.off + 16 * slab + (lane & 15);
  const uint32_t qrow = smem_u32(ls.qs) + R * 128;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int col = kk * 16 + (lane >> 4) * 8;
    ldsm_x4(qf[kk], qrow + (col >> 6) * (ls.qrows * 128) + ((((col & 63) >> 3) ^ (R & 7)) << 4));
  }
  acc.reset();
  const int n_keys = (n_in + 31) & ~31;
  for (int k0 = 0; k0 < n_keys; k0 += 32)
    consume_keys<D, 32>(acc, qf, smem_u32(ls.ks + (k0 / kBN) * kT), smem_u32(ls.vs + (k0 / kBN) * kT), k0 % kBN, k0,
                        n_in, p.scale_log2, lane);
}

// After the dependency wait: thread 0 expects the cached rows, and each box
// token's thread (its block position in `pos`) fetches the token's g cached A_out
// rows (contiguous in the cache) as one bulk copy and its L_out entries by
// cp.async.  A position out of range is recorded and its rows write nothing (the
// copy reads block row 0 so that the byte count holds).
template <int D>
__device__ __forceinline__ void lean_fetch(const Params& p, const LeanSmem<D>& ls, uint64_t* bars, int hk, int in0,
                                           int n_in, const LeanRows& lr, int pos, int tid) {
  const int g = p.g;
  if (tid == 0) mbar_arrive_expect_tx(&bars[1], lr.ntok * g * D * 4);
  const int t = lean_tok(tid);
  if (t >= 0 && t < lr.ntok) {
    const bool good = pos >= 0 && pos < n_in;
    if (!good) record_status(kDevBadIndex);
    const size_t ce = static_cast<size_t>(in0 + (good ? pos : 0)) * p.hq + hk * g;
    bulk_load_1d(ls.ca + t * g * D, p.cache_a + ce * D, g * D * 4, &bars[1]);
    for (int j = 0; j < g; ++j) cp_async_4(ls.cl + t * g + j, p.cache_l + ce + j);
    cp_async_commit();
    ls.pos[t] = good ? pos : -1;
  }
}

// A CTA whose group recomputes after all: the copies it issued early land before
// the streaming path reuses the shared memory.  Every thread calls it (it has a
// CTA barrier).
__device__ __forceinline__ void lean_drain(uint64_t* bars, int tid) {
  lean_wait(&bars[0], tid);
  lean_wait(&bars[1], tid);
  cp_async_wait_all();
  __syncthreads();
}

// Merge of warp slab `slab` with its cached rows, written to A_full / L_full.
template <int D>
__device__ __forceinline__ void lean_merge(const Params& p, const LeanSmem<D>& ls, const LeanRows& lr,
                                           const Acc<D>& acc, int slab, int lane, int q0, int hk) {
  const int g = p.g;
  // Merge weights of the thread's two rows first (independent chains), then each
  // row's columns: all of its cached values are loaded before any store (the loads
  // would otherwise wait behind the stores of earlier columns).
  float wo[2], wz[2], lf[2];
  int er[2], rr[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float z = quad_sum(acc.l[i]);
    const int R = lr.off + 16 * slab + (lane >> 2) + 8 * i;
    const int tt = R / g;
    rr[i] = R;
    er[i] = (R - lr.off < lr.nr && ls.pos[tt] >= 0) ? (q0 + lr.tok_lo + tt) * p.hq + hk * g + (R - tt * g) : -1;
    const float li2 = z > 0.f ? acc.m[i] + lg2_approx(z) : kNegInf;
    const float lo_nat = ls.cl[R];
    const float lo2 = lo_nat == kNegInf ? kNegInf : lo_nat * kLog2e;
    const float m2 = fmaxf(lo2, li2);
    float w_o = 0.f, w_i = 0.f, lf2 = kNegInf;
    if (m2 != kNegInf) {
      w_o = lo2 == kNegInf ? 0.f : ex2(lo2 - m2);
      w_i = li2 == kNegInf ? 0.f : ex2(li2 - m2);
      const float inv = rcp_approx(w_o + w_i);
      lf2 = m2 + lg2_approx(w_o + w_i);
      w_o *= inv;
      w_i *= inv;
    }
    wo[i] = w_o;
    wz[i] = z > 0.f ? w_i * rcp_approx(z) : 0.f;  // A_in = O / z
    lf[i] = lf2 == kNegInf ? kNegInf : lf2 * kLn2;
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (er[i] < 0) continue;
    const float* crow = ls.ca + rr[i] * D + 2 * (lane & 3);
    float2 ao[D / 8];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) ao[n] = *reinterpret_cast<const float2*>(crow + n * 8);
    __nv_bfloat16* dst = p.a_full + static_cast<size_t>(er[i]) * D + 2 * (lane & 3);
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<__nv_bfloat162*>(dst + n * 8) = __floats2bfloat162_rn(
          fmaf(wo[i], ao[n].x, wz[i] * acc.o[n][2 * i]), fmaf(wo[i], ao[n].y, wz[i] * acc.o[n][2 * i + 1]));
    if ((lane & 3) == 0 && p.l_full) p.l_full[er[i]] = lf[i];
  }
}

// The lean branch: wait for the inputs and the cached rows, then each warp
// attends and merges its slabs.  Every thread of the CTA calls it (it has a CTA
// barrier).
template <int D>
__device__ __forceinline__ void lean_finish(const Params& p, const LeanSmem<D>& ls, uint64_t* bars,
                                            const LeanRows& lr, int q0, int hk, int n_in, int tid, int nthreads) {
  const bool in_ok = lean_wait(&bars[0], tid);
  const bool ok = lean_wait(&bars[1], tid);
  cp_async_wait_all();  // the L_out entries this thread fetched
  if (!__syncthreads_and(ok && in_ok)) return;
  const int lane = tid & 31;
  for (int slab = tid >> 5; 16 * slab < lr.nr; slab += nthreads / 32) {
    Acc<D> acc;
    lean_attend<D>(p, ls, lr, slab, lane, n_in, acc);
    lean_merge<D>(p, ls, lr, acc, slab, lane, q0, hk);
  }
}

}  // namespace fb
