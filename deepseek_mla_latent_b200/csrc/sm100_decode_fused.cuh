// sm100_decode_fused.cuh -- a decode step's attention, split merge and output projection in one
// kernel ("Naive vs Absorb Attention Implementations in DeepSeek-V3", section "Absorb Path
// Execution": the score and latent value einsums, then the last einsum out = o_lat . W_v^T, with
// o_lat the log-sum-exp merge of the split partials).
//
// The grid is the attention kernel's (one CTA pair per (row, split) unit, all resident at once:
// one CTA per SM and no more CTAs than SMs).  After its unit, each CTA
//   1. makes its outputs visible (the value CTA waits until its partial stores have completed),
//   2. starts the TMA copy of W_v[h] for its first projection item into its now idle shared
//      memory (128 KB), so the weight stream overlaps the other units' tails,
//   3. arrives on a grid-wide counter and waits (bounded) until every CTA has arrived, i.e.
//      every partial of every row is in memory,
//   4. merges the split partials of its items (h, 16 query rows) into the B operand and runs the
//      projection's 32 tcgen05 products (M = 128 value rows, N = 16, K = 512), and stores out,
//   5. counts itself out; the last CTA out sets both counters back to zero.
// Items go to score CTAs first (their roles end several microseconds before the value CTAs').
// The merge and the products are merge_proj_kernel's, in the same order, so the result equals
// mla_attn_decode_out's bit for bit.
#pragma once

#include "sm100_merge_proj.cuh"

namespace mla {
namespace sm100 {

struct FusedParams {
  uint32_t* ctrl;          // [2] arrivals, departures: zero before a call, zero again after it
  int n_items;             // heads * ceil(n_q / 16)
  int row_tiles;           // ceil(n_q / 16)
  const __nv_bfloat16* part_o;
  const float* part_ml;
  int num_splits;
  int n_q;
  int heads;
  __nv_bfloat16* out;      // [n_q, heads, 128]
};

// Shared memory of the tail: W_v[h] (eight 16 KB K chunks), the B operand, the merge weights
// and row factors, barriers.  It lies below both roles' barrier areas.
struct FusedTailSmem {
  static constexpr int kW = 8 * 128 * 128;
  static constexpr int kOffB = kW;
  static constexpr int kOffWt = kOffB + 8 * kMpRows * 128;
  static constexpr int kOffInv = kOffWt + kMpMaxSplits * kMpRows * 4;
  static constexpr int kOffFlag = kOffInv + kMpRows * 4;
  static constexpr int kOffBars = kOffFlag + 64;
  static constexpr int kEnd = kOffBars + 64;
};
static_assert(FusedTailSmem::kEnd <= ValueLayout::kOffBars && FusedTailSmem::kEnd <= ScoreLayout::kOffBars,
              "the tail's shared memory overlaps a role's barriers");

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fused_tail(uint8_t* smem, uint32_t tmem, const CUtensorMap* tmap_w,
                                           const FusedParams& f) {
  using L = FusedTailSmem;
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id(), rank = ptx::cluster_rank();
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + L::kOffBars);   // W_v[h] landed
  uint64_t* done = wfull + 1;                                           // the products finished
  volatile int* flag = reinterpret_cast<volatile int*>(smem + L::kOffFlag);
  float* wt = reinterpret_cast<float*>(smem + L::kOffWt);
  float* inv_s = reinterpret_cast<float*>(smem + L::kOffInv);
  const int total = (int)gridDim.x, pairs = total >> 1;
  const int first = rank == 0 ? (int)(blockIdx.x >> 1) : pairs + (int)(blockIdx.x >> 1);

  // 1. this CTA's outputs are in memory: the partial stores of the value CTA's epilogue warps
  // (each lane 0 issued its own bulk group) have completed, and every thread's generic stores
  // (the score CTA's (m, l) pairs) are ordered before the arrival below
  if (lane == 0) {
    ptx::bulk_wait_all();
    ptx::fence_proxy_async_global();
  }
  __threadfence();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // 2. barriers of the tail (the role's shared memory is idle now) and the first item's weights
  if (threadIdx.x == 0) {
    ptx::mbar_init(wfull, 1);
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // W_v[h] of an item: one 3-D copy, the eight 64-column K chunks as the map's third axis
  int issued = 0;   // weight copies thread 0 started
  auto load_w = [&](int item) {
    const int h = item / f.row_tiles;
    ptx::mbar_arrive_expect_tx(wfull, L::kW);
    ptx::tma_load_3d(smem, tmap_w, wfull, 0, h * 256 + 128, 0);
    ++issued;
  };
  // (a shared-memory base off the swizzle's 1024-byte alignment has already been reported by the
  // attention set-up; the tail then stores nothing)
  const bool aligned = (ptx::smem_u32(smem) & 1023u) == 0;
  if (threadIdx.x == 0 && aligned && first < f.n_items) load_w(first);
  // 3. the grid-wide hand-off: every CTA's partials are in memory once all have arrived
  if (threadIdx.x == 0) {
    atomicAdd(f.ctrl, 1u);
    bool ok = true;
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(f.ctrl) < (uint32_t)total) {
      __nanosleep(64);
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        raise_error(kErrTimeoutPeer);
        ok = false;
        break;
      }
    }
    *flag = (ok && aligned) ? 1 : 0;
  }
  __syncthreads();
  const bool go = *flag != 0;

  // 4. the projection items of this CTA
  const int64_t split_stride = (int64_t)f.n_q * f.heads;
  int used = 0;
  for (int item = first; go && item < f.n_items; item += total, ++used) {
    const int h = item / f.row_tiles, n0 = (item % f.row_tiles) * kMpRows;
    if (used > 0) {
      // the previous item's products have read the weights and the B operand
      if (threadIdx.x == 0) load_w(item);
    }
    // merge weights: warp w handles rows w, w + 10
    for (int r = (int)warp; r < kMpRows; r += kAttnThreads / 32) {
      const int64_t n = n0 + r;
      if (n >= f.n_q) continue;   // warp-uniform
      const float2* ml = reinterpret_cast<const float2*>(f.part_ml) + n * f.heads + h;
      float M, inv;
      const float w_lane = merge_weights(ml, split_stride, f.num_splits, (int)lane, M, inv);
      for (int s = (int)lane; s < f.num_splits; s += 32) {
        float w = w_lane;
        if (s >= 32) {
          const float2 x = __ldcg(ml + s * split_stride);
          w = x.x == -INFINITY ? 0.f : exp2f(x.x - M);
        }
        wt[s * kMpRows + r] = w;
      }
      if (lane == 0) inv_s[r] = inv;
    }
    __syncthreads();
    // merge (row r, 16-byte column group g) items into the B operand
    const int64_t step = split_stride * 512 / 8;
    constexpr int kInFlight = 16;
    for (int it = (int)threadIdx.x; it < kMpRows * 64; it += kAttnThreads) {
      const int r = it >> 6, g = it & 63;
      uint4 o = make_uint4(0, 0, 0, 0);
      if (n0 + r < f.n_q) {
        const uint4* src = reinterpret_cast<const uint4*>(f.part_o + (((int64_t)n0 + r) * f.heads + h) * 512) + g;
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = 0.f;
        for (int s0 = 0; s0 < f.num_splits; s0 += kInFlight) {
          uint4 v[kInFlight];
#pragma unroll
          for (int s = 0; s < kInFlight; ++s)
            if (s0 + s < f.num_splits) v[s] = __ldcg(src + (s0 + s) * step);
#pragma unroll
          for (int s = 0; s < kInFlight; ++s)
            if (s0 + s < f.num_splits) {
              const float w = wt[(s0 + s) * kMpRows + r];
              if (w != 0.f) merge_acc(a, w, v[s]);
            }
        }
        const float inv = inv_s[r];
        o.x = ptx::pack_bf16x2(a[0] * inv, a[1] * inv);
        o.y = ptx::pack_bf16x2(a[2] * inv, a[3] * inv);
        o.z = ptx::pack_bf16x2(a[4] * inv, a[5] * inv);
        o.w = ptx::pack_bf16x2(a[6] * inv, a[7] * inv);
      }
      *reinterpret_cast<uint4*>(smem + L::kOffB + (g >> 3) * (kMpRows * 128) + r * 128 + (((g & 7) ^ (r & 7)) << 4)) = o;
    }
    ptx::fence_async_smem();
    __syncthreads();
    if (warp == 1) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kMpRows, false, false);
      const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(wfull, (uint32_t)(used & 1), kErrTimeoutTmaFull));
      if (ok) {
        ptx::tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          const uint32_t a = ptx::smem_u32(smem + k * 128 * 128), b = ptx::smem_u32(smem + L::kOffB + k * kMpRows * 128);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            if (ptx::elect_one())
              ptx::mma_ss(tmem, ptx::smem_desc(a + ks * 32, 16, 1024, ptx::kSwizzle128),
                          ptx::smem_desc(b + ks * 32, 16, 1024, ptx::kSwizzle128), idesc, (k | ks) ? 1u : 0u);
            __syncwarp();
          }
        }
      }
      if (ptx::elect_one()) ptx::mma_commit(done);
      __syncwarp();
    }
    if (warp < 4) {
      // out[n, h, d]: TMEM lane d (value row), column n - n0
      const bool ok = ptx::mbar_wait(done, (uint32_t)(used & 1), kErrTimeoutMma);
      ptx::tc_fence_after();
      if (ok) {
        uint32_t rr[16];
        ptx::tmem_ld16(tmem + ((warp * 32) << 16), rr);
        ptx::tmem_wait_ld();
        const int d = (int)(warp * 32 + lane);
#pragma unroll
        for (int j = 0; j < kMpRows; ++j) {
          const int64_t n = n0 + j;
          if (n < f.n_q) f.out[(n * f.heads + h) * 128 + d] = __float2bfloat16_rn(__uint_as_float(rr[j]));
        }
      }
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  // every weight copy this CTA started has landed before its shared memory goes away (the ones
  // the products consumed have; after a failed hand-off the first one is still to be waited for)
  if (threadIdx.x == 0 && issued > 0) ptx::mbar_wait(wfull, (uint32_t)((issued - 1) & 1), kErrTimeoutDrain);
  // 5. count out; the last CTA out leaves both counters at zero for the next call
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t old = atomicAdd(f.ctrl + 1, 1u);
    if (old == (uint32_t)total - 1) {
      f.ctrl[0] = 0;
      f.ctrl[1] = 0;
      __threadfence();
    }
  }
}

// The fused decode kernel: the attention kernel's CTA pairs, then the tail above.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmap_kv_score, const __grid_constant__ CUtensorMap tmap_pe,
                        const __grid_constant__ CUtensorMap tmap_qpe, const __grid_constant__ CUtensorMap tmap_kv_value,
                        const __grid_constant__ CUtensorMap tmap_qabs, const __grid_constant__ CUtensorMap tmap_out,
                        const __grid_constant__ CUtensorMap tmap_w, const AttnParams p, const FusedParams f) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t tmem = attn_unit<false>(smem, &tmap_kv_score, &tmap_pe, &tmap_qpe, &tmap_kv_value, &tmap_qabs,
                                         &tmap_out, p);
  fused_tail(smem, tmem, &tmap_w, f);
  attn_teardown(tmem);
}

}  // namespace sm100
}  // namespace mla
