// Work order of the two-tile kernel.  With the similarity gate half of a video
// block's heads may recompute (87 key chunks per CTA) while the others reuse (13):
// launched in head order, the long CTAs that start in the last wave leave most
// SMs idle at the end.  This one-CTA pass takes every head's decision (the same
// head_recompute the attention kernel evaluates, after the similarity scores are
// written) and lists the work items -- (sequence, head, 256-row pair) -- with the
// recomputing ones first, in index order within each class; the attention kernel's
// CTA i then takes item order[i].
#pragma once

#include "fb_kernels.cuh"

namespace fb {

constexpr int kOrderThreads = 1024;

__global__ void __launch_bounds__(kOrderThreads) order_kernel(const __grid_constant__ Params p, int* order) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_cnt[kOrderThreads];
  const int tid = threadIdx.x;
  const int pairs = p.tiles;
  const int n = p.num_seqs * p.hq * pairs;
  const int per = (n + kOrderThreads - 1) / kOrderThreads;  // contiguous items of this thread
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int heavy = 0;
  for (int i = i0; i < i1; ++i) heavy += head_recompute(p, i / pairs / p.hq, i / pairs % p.hq) ? 1 : 0;
  s_cnt[tid] = heavy;
  __syncthreads();
  // inclusive scan of the per-thread counts (Hillis-Steele)
  for (int off = 1; off < kOrderThreads; off <<= 1) {
    const int v = tid >= off ? s_cnt[tid - off] : 0;
    __syncthreads();
    s_cnt[tid] += v;
    __syncthreads();
  }
  const int n_heavy = s_cnt[kOrderThreads - 1];
  int h_pos = s_cnt[tid] - heavy;  // heavy items before this thread's
  int l_pos = n_heavy + (i0 - h_pos);  // light items before: i0 minus the heavy ones
  for (int i = i0; i < i1; ++i) {
    if (head_recompute(p, i / pairs / p.hq, i / pairs % p.hq))
      order[h_pos++] = i;
    else
      order[l_pos++] = i;
  }
}

}  // namespace fb
