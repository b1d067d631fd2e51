// Sparse-residual key layout (FlashBlock, "Estrategias de Reutilizacion
// Adaptativa", third bullet: the keys a sparse pattern does not select form the
// out-of-block set whose contribution is cached).  Per sequence b, the selected
// prefix keys join the block's keys -- J_in' = block keys, then the selected keys
// in increasing order -- and the others form the residual prefix J_out' (order
// kept).  The attention kernels then run unchanged on (J_out', J_in').
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
  __nv_bfloat16* k_res;
  __nv_bfloat16* v_res;
  __nv_bfloat16* k_ext;
  __nv_bfloat16* v_ext;
  int* cu_out_res;  // optional: cu_out - cu_sel
  int* cu_in_ext;   // optional: cu_in + cu_sel
};

// blockIdx.y = sequence; the x-blocks stride over (token, 16-byte piece) items of
// the sequence's prefix then block rows.  Each prefix token finds its rank among
// the selected positions by binary search.
__global__ void __launch_bounds__(256) sparse_layout_kernel(const SparseParams p) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int o0 = p.cu_out[b], n_out = p.cu_out[b + 1] - o0;
  const int i0 = p.cu_in[b], n_in = p.cu_in[b + 1] - i0;
  const int s0 = p.cu_sel[b], n_sel = p.cu_sel[b + 1] - s0;
  // The whole CTA checks the ranges, then the selection (strictly increasing
  // prefix positions), one element per thread per pass.
  int ok = o0 >= 0 && n_out >= 0 && o0 + n_out <= p.total_out && i0 >= 0 && n_in >= 0 && i0 + n_in <= p.total_in &&
           s0 >= 0 && n_sel >= 0 && s0 + n_sel <= p.total_sel && n_sel <= n_out;
  for (int k = threadIdx.x; ok && k < n_sel; k += blockDim.x) {
    const int v = p.sel[s0 + k];
    ok = v >= 0 && v < n_out && (k == 0 || v > p.sel[s0 + k - 1]);
  }
  ok = __syncthreads_and(ok);
  if (!ok) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(kDevBadIndex);
    return;
  }
  const int r0 = o0 - s0;  // J_out' of b starts here
  const int e0 = i0 + s0;  // J_in' of b starts here
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (p.cu_out_res) p.cu_out_res[b] = r0;
    if (p.cu_in_ext) p.cu_in_ext[b] = e0;
    if (b == p.num_seqs - 1) {
      if (p.cu_out_res) p.cu_out_res[b + 1] = p.cu_out[b + 1] - p.cu_sel[b + 1];
      if (p.cu_in_ext) p.cu_in_ext[b + 1] = p.cu_in[b + 1] + p.cu_sel[b + 1];
    }
  }
  const int vec = p.hkv * p.d / 8;  // 16-byte pieces per token row
  const long items = static_cast<long>(n_out + n_in) * vec;
  for (long it = blockIdx.x * 256l + threadIdx.x; it < items; it += static_cast<long>(gridDim.x) * 256) {
    const int tok = static_cast<int>(it / vec);
    const int c = static_cast<int>(it % vec) * 8;
    const uint4* sk;
    const uint4* sv;
    uint4* dk;
    uint4* dv;
    if (tok < n_out) {
      int lo = 0, hi = n_sel;  // rank = number of selected positions below tok
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (p.sel[s0 + mid] < tok) lo = mid + 1; else hi = mid;
      }
      const size_t src = static_cast<size_t>(o0 + tok) * p.hkv * p.d + c;
      sk = reinterpret_cast<const uint4*>(p.k_out + src);
      sv = reinterpret_cast<const uint4*>(p.v_out + src);
      const bool selected = lo < n_sel && p.sel[s0 + lo] == tok;
      const size_t dst = selected ? static_cast<size_t>(e0 + n_in + lo) * p.hkv * p.d + c
                                  : static_cast<size_t>(r0 + tok - lo) * p.hkv * p.d + c;
      dk = reinterpret_cast<uint4*>((selected ? p.k_ext : p.k_res) + dst);
      dv = reinterpret_cast<uint4*>((selected ? p.v_ext : p.v_res) + dst);
    } else {
      const int t = tok - n_out;
      const size_t src = static_cast<size_t>(i0 + t) * p.hkv * p.d + c;
      const size_t dst = static_cast<size_t>(e0 + t) * p.hkv * p.d + c;
      sk = reinterpret_cast<const uint4*>(p.k_in + src);
      sv = reinterpret_cast<const uint4*>(p.v_in + src);
      dk = reinterpret_cast<uint4*>(p.k_ext + dst);
      dv = reinterpret_cast<uint4*>(p.v_ext + dst);
    }
    *dk = *sk;
    *dv = *sv;
  }
}

}  // namespace fb
