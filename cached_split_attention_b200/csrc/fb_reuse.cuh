// Lean reuse path of the fused FlashBlock step (sm_100a).
//
// On a reuse step the out-of-block partial (A_out, L_out) comes from the cache, so
// the only attention left is the block's own: every active query row against the
// block's B keys (bidirectional), followed by the log-space merge with the cached
// row (FlashBlock, "Mecanismo Central": the stored values are reused instead of
// reading the prefix K/V again).  That is a few MB per call and a short chain of
// dependent loads, so when no head of a group (sequence, kv-head, row tile)
// recomputes, the streaming kernels hand the group to this path instead of their
// TMA pipeline, cluster and merge phases.  The group's CTAs share its rows (16 per
// warp) and each runs:
//
//   loads      by TMA, completed on one mbarrier: the block K/V of the kv-head as
//              64-row tensor-map boxes (whole 64-key chunks; keys past the block
//              are masked), each row's Q as a 1-D bulk copy, and -- as soon as the
//              row's block position (q_rows) is back -- its cached A_out entry
//              (1-D bulk) and L_out;
//   attention  S = Q K^T and O = P V with mma.sync (bf16 in, fp32 accumulate),
//              online softmax in base 2 (the streaming kernel's inner loop);
//   merge      in registers: A_full = w_out A_out + w_in A_in, L_full =
//              logaddexp(L_out, L_in), written as bf16 / fp32.
//
// K and V sit in shared memory in the 128-byte swizzled layout of the warp-MMA
// kernel's stages (64-key chunks), so the same inner loop serves both.  Keys past
// the block's end are masked (rows past the tensor's end arrive as zeros, rows of
// the next sequence are finite).  Blocks of up to kMaxKeys keys take
// this path (the host plan checks max_kv_in and the shared memory it needs);
// longer blocks are real contractions and stay on the streaming pipelines.
//
// Included by fb_kernels.cuh after the helpers it shares with the warp-MMA kernel
// (Params, swz, Acc, consume_keys) and before the kernels that call it.
#pragma once

namespace fb {
namespace reuse {

constexpr int kMaxKeys = 128;  // block keys a CTA holds: two 64-key chunks

// Shared memory of the lean path for `chunks` 64-key chunks and `rows` rows (a
// multiple of 16), after the 1024-byte alignment of the kernel's base.
__host__ __device__ constexpr int tile_bytes(int d) { return kBN * d * 2; }
__host__ __device__ constexpr int q_stride(int d) { return d + 8; }  // padded bf16 Q row
__host__ __device__ constexpr int c_stride(int d) { return d + 4; }  // padded fp32 cache row
__host__ __device__ constexpr int smem_bytes(int d, int chunks, int rows) {
  // K, V chunks; Q rows; cache A rows; cache L; output entry of each row; the barrier
  return 2 * chunks * tile_bytes(d) + rows * q_stride(d) * 2 + rows * c_stride(d) * 4 + rows * 4 + rows * 4 + 16;
}

}  // namespace reuse

// Rows [r0, r0 + nr) of group (b, hk) -- row rho = (token rho / g, q-head hk*g +
// rho % g) of the sequence's packed active tokens -- with the block keys of b.
// Every thread of the CTA calls it (it has CTA barriers); `smem` is the kernel's
// 1024-byte aligned dynamic shared memory.
// Block position of the lean row thread `tid` owns among rows [r0, r0 + nr) (-1:
// none).  Read from q_rows before the kernel waits for the previous kernel of the
// stream (index arrays are not written by any kernel that lets this one start
// early); the caller has checked the sequence's ranges against the host totals.
__device__ __forceinline__ int lean_pos(const Params& p, int q0, int r0, int nr, int tid) {
  if (tid >= nr) return -1;
  const int tok = (r0 + tid) / p.g;
  return p.q_rows ? p.q_rows[q0 + tok] : tok;
}

template <int D>
__device__ __forceinline__ void lean_reuse(const Params& p, uint8_t* smem, int b, int hk, int q0, int in0, int n_in,
                                           int r0, int nr, int pos_pre, int tid, int nthreads) {
  constexpr int kT = reuse::tile_bytes(D);
  constexpr int kQS = reuse::q_stride(D);
  constexpr int kCS = reuse::c_stride(D);
  const int g = p.g;
  const int nch = p.reuse_chunks;
  const int nr16 = (nr + 15) & ~15;
  uint8_t* ks = smem;
  uint8_t* vs = smem + nch * kT;
  __nv_bfloat16* q_s = reinterpret_cast<__nv_bfloat16*>(smem + 2 * nch * kT);
  float* ca_s = reinterpret_cast<float*>(smem + 2 * nch * kT + nr16 * kQS * 2);
  float* cl_s = ca_s + nr16 * kCS;
  int* fe_s = reinterpret_cast<int*>(cl_s + nr16);  // output entry of each row; -1: no output
  uint64_t* bar = reinterpret_cast<uint64_t*>(fe_s + nr16);
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int used = (n_in + kBN - 1) / kBN;  // 64-key chunks holding the block

  // One thread per row has its block position (read before the dependency wait);
  // thread 0 arms the barrier: one arrival per row, one for the block K/V.
  int pos = pos_pre, fe = -1;
  if (tid < nr) {
    const int rho = r0 + tid;
    const int tok = rho / g;
    fe = (q0 + tok) * p.hq + hk * g + (rho - tok * g);
  }
  if (tid == 0) {
    mbar_init(bar, nr + 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {  // block K/V of kv-head hk, whole 64-key chunks (keys past the block are masked)
    mbar_arrive_expect_tx(bar, 2 * used * kT);
    for (int c = 0; c < used; ++c) {
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_2d_plain(ks + c * kT + hh * (kBN * 128), &p.tm_k_lean, bar, hk * D + hh * 64, in0 + c * kBN);
        tma_load_2d_plain(vs + c * kT + hh * (kBN * 128), &p.tm_v_lean, bar, hk * D + hh * 64, in0 + c * kBN);
      }
    }
  }
  if (tid < nr) {  // the row's Q, then (once its position is back) its cache entry
    mbar_expect_tx(bar, D * 2);
    bulk_load_1d(q_s + tid * kQS, p.q + static_cast<size_t>(fe) * D, D * 2, bar);
    if (pos < 0 || pos >= n_in) {
      record_status(kDevBadIndex);
      fe = -1;
      mbar_arrive(bar);
    } else {
      const size_t ce = static_cast<size_t>(in0 + pos) * p.hq + (fe % p.hq);
      mbar_arrive_expect_tx(bar, D * 4);
      bulk_load_1d(ca_s + tid * kCS, p.cache_a + ce * D, D * 4, bar);
      cp_async_4(cl_s + tid, p.cache_l + ce);
      cp_async_commit();
    }
  } else if (tid < nr16) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c) *reinterpret_cast<uint4*>(q_s + tid * kQS + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  if (tid < nr16) fe_s[tid] = fe;
  // every thread waits for the copies; on a timeout (never expected) the copies
  // still in flight get a second bounded wait before the CTA moves on
  bool ok = mbar_wait(bar, 0);
  if (!ok) {
    if (tid == 0) record_status(kDevTimeout);
    mbar_wait(bar, 0);
  }
  cp_async_wait_all();  // the row's L_out
  __syncthreads();
  if (!ok) return;

  const int n_keys = (n_in + 31) & ~31;
  for (int slab = warp; slab * 16 < nr; slab += nthreads / 32) {
    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      ldsm_x4(qf[kk], smem_u32(q_s + (16 * slab + (lane & 15)) * kQS + kk * 16 + (lane >> 4) * 8));
    Acc<D> acc;
    acc.reset();
    for (int k0 = 0; k0 < n_keys; k0 += 32) {
      const uint32_t kb = smem_u32(ks + (k0 / kBN) * kT);
      const uint32_t vb = smem_u32(vs + (k0 / kBN) * kT);
      consume_keys<D, 32>(acc, qf, kb, vb, k0 % kBN, k0, n_in, p.scale_log2, lane);
    }
    // Merge weights of the thread's two rows first (independent chains), then
    // each row's columns: all of its cached values are loaded before any store
    // (the loads would otherwise wait behind the stores of earlier columns).
    float wo[2], wz[2], lf[2];
    int er[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float z = quad_sum(acc.l[i]);
      const int r = 16 * slab + (lane >> 2) + 8 * i;
      er[i] = fe_s[r];
      const float li2 = z > 0.f ? acc.m[i] + lg2_approx(z) : kNegInf;
      const float lo_nat = cl_s[r];
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
      const float* crow = ca_s + (16 * slab + (lane >> 2) + 8 * i) * kCS + 2 * (lane & 3);
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
}

// The rows of a served group that CTA `split` of its S takes: whole 16-row warp
// slabs, dealt out as evenly as the slabs allow.
__device__ __forceinline__ void lean_rows(int nrows, int split, int S, int& r0, int& nr) {
  const int slabs = (nrows + 15) / 16;
  const int per = (slabs + S - 1) / S;
  r0 = min(nrows, split * per * 16);
  nr = min(nrows, (split + 1) * per * 16) - r0;
}

}  // namespace fb
