// Sparse-residual key layout (FlashBlock, "Estrategias de Reutilizacion
// Adaptativa", third bullet: the keys a sparse pattern does not select form the
// out-of-block set whose contribution is cached).  Per sequence b, the selected
// prefix keys join the block's keys -- J_in' = block keys, then the selected keys
// in increasing order -- and the others form the residual prefix J_out'.  The
// residual is not copied: the selected prefix tokens are marked in a bitmask that
// the prefix pass of every attention kernel consults (fb_problem.kv_out_skip), so
// this pass moves only the block rows and the selected rows (a few MB) instead of
// the whole prefix.
#pragma once

#include "fb_device.cuh"
#include "fb_kernels.cuh"

namespace fb {

struct SparseParams {
  int num_seqs, hkv, d, total_out, total_in, total_sel;
  const int* cu_out;
  const int* cu_in;
  const int* cu_sel;
  const int* sel;
  const __nv_bfloat16* k_out;
  const __nv_bfloat16* v_out;
  const __nv_bfloat16* k_in;
  const __nv_bfloat16* v_in;
  __nv_bfloat16* k_ext;
  __nv_bfloat16* v_ext;
  uint32_t* skip;   // bit t: prefix token t selected
  int* cu_in_ext;   // optional: cu_in + cu_sel
};

// blockIdx.y = sequence; the x-blocks stride over (row, 16-byte piece) items of the
// sequence's J_in' rows: its block rows, then its selected prefix rows.  A copy of a
// selected row checks its own entry against the one before it (a strictly
// increasing selection is one whose neighbours all increase), in the round trip
// that fetches its address, and writes nothing when they do not.  The first
// x-block checks the whole selection and writes the skip bits of the sequence's
// prefix tokens: cleared (a word shared with a neighbouring sequence only in this
// sequence's bits, by atomics), then -- for a good selection -- the selected ones
// set; it also records a bad selection and writes the J_in' offsets.
__global__ void __launch_bounds__(256) sparse_layout_kernel(const SparseParams p) {
  pdl_wait();
  // no early launch of the next kernel: it may read what this one writes (index
  // arrays, K/V) before its own dependency wait
  const int b = blockIdx.y;
  const int o0 = p.cu_out[b], n_out = p.cu_out[b + 1] - o0;
  const int i0 = p.cu_in[b], n_in = p.cu_in[b + 1] - i0;
  const int s0 = p.cu_sel[b], n_sel = p.cu_sel[b + 1] - s0;
  const bool ranges = o0 >= 0 && n_out >= 0 && o0 + n_out <= p.total_out && i0 >= 0 && n_in >= 0 &&
                      i0 + n_in <= p.total_in && s0 >= 0 && n_sel >= 0 && s0 + n_sel <= p.total_sel && n_sel <= n_out;
  if (!ranges) {  // the same in every thread
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(kDevBadIndex);
    return;
  }
  const int e0 = i0 + s0;  // J_in' of b starts here
  if (blockIdx.x == 0) {
    int ok = 1;
    for (int k = threadIdx.x; k < n_sel; k += blockDim.x) {
      const int v = p.sel[s0 + k];
      const int u = k == 0 ? -1 : p.sel[s0 + k - 1];
      ok &= v >= 0 && v < n_out && v > u;
    }
    if (n_out > 0) {
      const int w_lo = o0 >> 5, w_hi = (o0 + n_out - 1) >> 5;
      for (int w = w_lo + static_cast<int>(threadIdx.x); w <= w_hi; w += blockDim.x) {
        const int a = max(w * 32, o0) - w * 32, z = min(w * 32 + 32, o0 + n_out) - w * 32;  // b's bits [a, z)
        if (z - a == 32) {
          p.skip[w] = 0u;
        } else {
          atomicAnd(p.skip + w, ~(((1u << (z - a)) - 1u) << a));
        }
      }
    }
    ok = __syncthreads_and(ok);  // also: every bit cleared before any is set
    if (ok) {
      for (int k = threadIdx.x; k < n_sel; k += blockDim.x) {
        const int t = o0 + p.sel[s0 + k];
        atomicOr(p.skip + (t >> 5), 1u << (t & 31));
      }
      if (threadIdx.x == 0 && p.cu_in_ext) {
        p.cu_in_ext[b] = e0;
        if (b == p.num_seqs - 1) p.cu_in_ext[b + 1] = p.cu_in[b + 1] + p.cu_sel[b + 1];
      }
    } else if (threadIdx.x == 0) {
      record_status(kDevBadIndex);
    }
  }
  const int vec = p.hkv * p.d / 8;  // 16-byte pieces per token row
  const long items = static_cast<long>(n_in + n_sel) * vec;
  for (long it = blockIdx.x * 256l + threadIdx.x; it < items; it += static_cast<long>(gridDim.x) * 256) {
    const int row = static_cast<int>(it / vec);
    const int c = static_cast<int>(it % vec) * 8;
    size_t src;
    bool good = true;
    if (row < n_in) {
      src = static_cast<size_t>(i0 + row) * p.hkv * p.d + c;
    } else {
      const int k = row - n_in;
      const int v = p.sel[s0 + k];
      const int u = k == 0 ? -1 : p.sel[s0 + k - 1];
      good = v >= 0 && v < n_out && v > u;
      src = static_cast<size_t>(o0 + min(max(v, 0), n_out - 1)) * p.hkv * p.d + c;
    }
    const bool blk = row < n_in;
    const uint4 kv = *reinterpret_cast<const uint4*>((blk ? p.k_in : p.k_out) + src);
    const uint4 vv = *reinterpret_cast<const uint4*>((blk ? p.v_in : p.v_out) + src);
    if (!good) continue;
    const size_t dst = static_cast<size_t>(e0 + row) * p.hkv * p.d + c;
    *reinterpret_cast<uint4*>(p.k_ext + dst) = kv;
    *reinterpret_cast<uint4*>(p.v_ext + dst) = vv;
  }
}

}  // namespace fb
