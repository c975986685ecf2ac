// gather.cuh -- token-granular selection for sparse decode ("What is DeepSeek
// Sparse Attention (DSA)? A clear, modern explainer", section "How DSA works
// (conceptual)": exact attention over the shortlisted tokens only).
//
// The selected cache rows of sequence b, indices[b, 0 .. counts[b]-1] (any
// rows of the packed latent cache, any order), are copied into page b of a
// paged scratch cache: row i of the list goes to row b * page + i.  The paged
// attention kernels then attend to exactly those keys (block table entry b =
// page b, key count = counts[b]).  One warp per selected row; every lane issues
// its 16-byte loads of the latent row (and the rotary row) before its stores.
// A listed row outside the cache is written as zeros and raises bit 1<<7 of the
// device error word (as an out-of-cache page does for the paged calls).
#pragma once

#include "common.cuh"

namespace mla {
namespace gather {

constexpr int kWarps = 8;

// kv_vec / pe_vec: 16-byte vectors per latent / rotary row (at most 64 / 8 per lane pass).
__global__ void __launch_bounds__(kWarps * 32)
    select_rows_kernel(const uint4* __restrict__ kv, const uint4* __restrict__ pe, int64_t kv_rows,
                       const int* __restrict__ indices, int64_t index_stride, const int* __restrict__ counts,
                       int max_topk, int64_t page, int kv_vec, int pe_vec, uint4* __restrict__ kv_out,
                       uint4* __restrict__ pe_out, int* __restrict__ seqlens_out, int* __restrict__ table_out) {
  const int b = blockIdx.y;
  int n = __ldg(counts + b);
  n = n < 0 ? 0 : (n > max_topk ? max_topk : n);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    seqlens_out[b] = n;
    table_out[b] = b;
  }
  const int warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t i = (int64_t)blockIdx.x * kWarps + warp; i < n; i += (int64_t)gridDim.x * kWarps) {
    const int r = __ldg(indices + (int64_t)b * index_stride + i);
    const bool ok = r >= 0 && r < kv_rows;
    if (!ok && lane == 0) raise_error(kErrBadPage);
    const int64_t dst = (int64_t)b * page + i;
    uint4 x[2], y;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = lane + 32 * k;
      x[k] = (ok && v < kv_vec) ? __ldg(kv + (int64_t)r * kv_vec + v) : zero;
    }
    y = (ok && lane < pe_vec) ? __ldg(pe + (int64_t)r * pe_vec + lane) : zero;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = lane + 32 * k;
      if (v < kv_vec) kv_out[dst * kv_vec + v] = x[k];
    }
    if (lane < pe_vec) pe_out[dst * pe_vec + lane] = y;
  }
}

}  // namespace gather
}  // namespace mla
