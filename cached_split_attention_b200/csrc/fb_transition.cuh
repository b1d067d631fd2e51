// Block transition (FlashBlock, "Mecanismo Central": a finished block's tokens stop
// being denoised and become context, i.e. part of the next block's out-of-block
// set J_out).  For every sequence b the grown prefix is J_out(b) followed by the
// finished block's K/V, J_in(b), in block order:
//     J_out'(b) = J_out(b) ++ J_in(b),   cu_out'[b] = cu_out[b] + cu_in[b].
// The next block brings new queries, so the FlashBlock cache is invalidated
// (fb_cache_invalidate) rather than extended.
#pragma once

#include "fb_device.cuh"
#include "fb_kernels.cuh"

namespace fb {

struct AppendParams {
  int num_seqs, hkv, d, total_out, total_in;
  int copy_prefix;  // 0: in place (one sequence; the prefix rows stay where they are)
  const int* cu_out;
  const int* cu_in;
  const __nv_bfloat16* k_out;
  const __nv_bfloat16* v_out;
  const __nv_bfloat16* k_in;
  const __nv_bfloat16* v_in;
  __nv_bfloat16* k_dst;
  __nv_bfloat16* v_dst;
  int* cu_dst;  // optional: cu_out + cu_in
};

// blockIdx.y = sequence; the x-blocks stride over (token, 16-byte piece) items of
// the sequence's prefix rows (when copied) then its block rows.
__global__ void __launch_bounds__(256) prefix_append_kernel(const AppendParams p) {
  pdl_wait();
  // no early launch of the next kernel: it may read what this one writes (index
  // arrays, K/V) before its own dependency wait
  const int b = blockIdx.y;
  const int o0 = p.cu_out[b], n_out = p.cu_out[b + 1] - o0;
  const int i0 = p.cu_in[b], n_in = p.cu_in[b + 1] - i0;
  const bool ok = o0 >= 0 && n_out >= 0 && o0 + n_out <= p.total_out && i0 >= 0 && n_in >= 0 &&
                  i0 + n_in <= p.total_in;
  if (!ok) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(kDevBadIndex);
    return;
  }
  const int n0 = o0 + i0;  // J_out'(b) starts here
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.cu_dst) {
    p.cu_dst[b] = n0;
    if (b == p.num_seqs - 1) p.cu_dst[b + 1] = p.cu_out[b + 1] + p.cu_in[b + 1];
  }
  const int vec = p.hkv * p.d / 8;  // 16-byte pieces per token row
  const int first = p.copy_prefix ? 0 : n_out;
  const long items = static_cast<long>(n_out + n_in - first) * vec;
  for (long it = blockIdx.x * 256l + threadIdx.x; it < items; it += static_cast<long>(gridDim.x) * 256) {
    const int tok = first + static_cast<int>(it / vec);
    const int c = static_cast<int>(it % vec) * 8;
    const size_t src = tok < n_out ? static_cast<size_t>(o0 + tok) * p.hkv * p.d + c
                                   : static_cast<size_t>(i0 + tok - n_out) * p.hkv * p.d + c;
    const size_t dst = static_cast<size_t>(n0 + tok) * p.hkv * p.d + c;
    const __nv_bfloat16* sk = tok < n_out ? p.k_out : p.k_in;
    const __nv_bfloat16* sv = tok < n_out ? p.v_out : p.v_in;
    *reinterpret_cast<uint4*>(p.k_dst + dst) = *reinterpret_cast<const uint4*>(sk + src);
    *reinterpret_cast<uint4*>(p.v_dst + dst) = *reinterpret_cast<const uint4*>(sv + src);
  }
}

}  // namespace fb
