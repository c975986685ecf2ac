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
//   4. merges the split partials of its items (h, 16 query rows) into the B operand -- each thread
//      loads its row's (m, l) pairs and its partials in one memory round trip -- and runs the
//      projection's 32 tcgen05 products (M = 128 value rows, N = 16, K = 512), and stores out,
//   5. counts itself out; the last CTA out sets both counters back to zero.
// Items go to score CTAs first (their roles end several microseconds before the value CTAs').
// The merge and the products are merge_proj_kernel's, in the same order, so the result equals
// mla_attn_decode_out's bit for bit.
#pragma once

#include "sm100_merge_proj.cuh"

namespace mla {
namespace sm100 {

// Splits the one-kernel step merges from registers (each thread holds all of them in flight).
constexpr int kMergeMaxSplitsFused = 12;

struct FusedParams {
  CUtensorMap tmap_part;   // the split partials as [splits][n_q][H][512] bf16, boxes [S][R][1][256]
  uint32_t* ctrl;          // [2] arrivals, departures: zero before a call, zero again after it
  int part_rows;           // R: rows of an item's partial copy (min(16, n_q))
  int n_items;             // heads * ceil(n_q / 16)
  int row_tiles;           // ceil(n_q / 16)
  const __nv_bfloat16* part_o;
  const float* part_ml;
  int num_splits;
  int n_q;
  int heads;
  __nv_bfloat16* out;      // [n_q, heads, 128]
};

// Shared memory of the tail: W_v[h] (eight 16 KB K chunks), the item's split partials (two TMA
// copies of [splits][rows][256 columns] bf16, at most 74 rows x splits in all), the B operand, the
// hand-off flag, barriers.  It lies below the score role's barrier area; on the value CTA it
// covers the value role's barriers, which nothing uses once the role has ended (every copy into
// that CTA and every arrival on its barriers completed before its epilogue).
struct FusedTailSmem {
  static constexpr int kW = 8 * 128 * 128;
  static constexpr int kMaxRowSplits = 74;                  // rows x splits of an item (all CTAs resident)
  static constexpr int kOffPart = kW;
  static constexpr int kPartHalf = kMaxRowSplits * 256 * 2;
  static constexpr int kOffB = kOffPart + 2 * kPartHalf;
  static constexpr int kOffFlag = kOffB + 8 * kMpRows * 128;
  static constexpr int kOffBars = kOffFlag + 64;
  static constexpr int kEnd = kOffBars + 64;
};
static_assert(FusedTailSmem::kEnd <= ScoreLayout::kOffBars && FusedTailSmem::kEnd <= kAttnSmem,
              "the tail's shared memory overlaps the score role's barriers");

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
  uint64_t* pfull = wfull + 2;                                          // the item's partials landed
  volatile int* flag = reinterpret_cast<volatile int*>(smem + L::kOffFlag);
  const int total = (int)gridDim.x, pairs = total >> 1;
  const int first = rank == 0 ? (int)(blockIdx.x >> 1) : pairs + (int)(blockIdx.x >> 1);

  // 0. every thread that touches global memory below has waited for the previous kernel (the
  // attention roles' MMA warps had no reason to)
  ptx::griddep_wait();
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
    ptx::mbar_init(pfull, 1);
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
    // the item's split partials into shared memory (two TMA copies: columns 0..255 and 256..511 of
    // [splits][rows n0 .. n0 + R)[head h]), while each thread loads its row's (m, l) pairs
    const int R = f.part_rows;
    const int part_half = f.num_splits * R * 256 * 2;
    if (threadIdx.x == 0) {
      ptx::mbar_arrive_expect_tx(pfull, 2 * part_half);
      ptx::tma_load_4d(smem + L::kOffPart, &f.tmap_part, pfull, 0, h, n0, 0);
      ptx::tma_load_4d(smem + L::kOffPart + part_half, &f.tmap_part, pfull, 256, h, n0, 0);
    }
    // merge (row r, 16-byte column groups g and g + 32) into the B operand: thread t < 256 takes row
    // t / 32 of a 8-row pass, with the arithmetic of merge_weights (row sum in the same order) and
    // of the merge kernels, so the result is the two-kernel path's bit for bit
    for (int r0 = 0; r0 < kMpRows; r0 += 8) {
      const int r = r0 + ((int)threadIdx.x >> 5), g0 = (int)threadIdx.x & 31;
      const bool active = threadIdx.x < 256;
      const bool valid = active && r < R && n0 + r < f.n_q;
      float2 ml[kMergeMaxSplitsFused];
      if (valid) {
        const float2* mlp = reinterpret_cast<const float2*>(f.part_ml) + ((int64_t)n0 + r) * f.heads + h;
#pragma unroll
        for (int sp = 0; sp < kMergeMaxSplitsFused; ++sp)
          if (sp < f.num_splits) ml[sp] = __ldcg(mlp + sp * split_stride);
      }
      const bool landed = ptx::mbar_wait(pfull, (uint32_t)(used & 1), kErrTimeoutTmaFull);
      if (active) {
        uint4 o[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        if (valid && landed) {
          float M = -INFINITY;
#pragma unroll
          for (int sp = 0; sp < kMergeMaxSplitsFused; ++sp)
            if (sp < f.num_splits) M = fmaxf(M, ml[sp].x);
          float a[2][8];
#pragma unroll
          for (int i = 0; i < 8; ++i) a[0][i] = a[1][i] = 0.f;
          // the row sum sum_s w_s l_s added in the order of the warp butterfly merge_weights uses
          // (xor 16, 8, 4, 2, 1 over lanes = splits; splits past the count hold 0)
          float x[16];
#pragma unroll
          for (int sp = 0; sp < 16; ++sp) x[sp] = 0.f;
#pragma unroll
          for (int sp = 0; sp < kMergeMaxSplitsFused; ++sp)
            if (sp < f.num_splits) {
              const float w = ml[sp].x == -INFINITY ? 0.f : exp2f(ml[sp].x - M);
              x[sp] = w * ml[sp].y;
              if (w != 0.f) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                  // column group g = g0 + 32k: columns 8g .. 8g + 7, in copy (8g) / 256
                  const int c = 8 * (g0 + 32 * k);
                  const uint8_t* src = smem + L::kOffPart + (c >> 8) * part_half + ((sp * R + r) * 256 + (c & 255)) * 2;
                  merge_acc(a[k], w, *reinterpret_cast<const uint4*>(src));
                }
              }
            }
#pragma unroll
          for (int o2 = 8; o2 >= 1; o2 >>= 1)
#pragma unroll
            for (int i = 0; i < o2; ++i) x[i] = x[i] + x[i + o2];
          const float inv = x[0] > 0.f ? 1.f / x[0] : 0.f;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            o[k].x = ptx::pack_bf16x2(a[k][0] * inv, a[k][1] * inv);
            o[k].y = ptx::pack_bf16x2(a[k][2] * inv, a[k][3] * inv);
            o[k].z = ptx::pack_bf16x2(a[k][4] * inv, a[k][5] * inv);
            o[k].w = ptx::pack_bf16x2(a[k][6] * inv, a[k][7] * inv);
          }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int g = g0 + 32 * k;
          *reinterpret_cast<uint4*>(smem + L::kOffB + (g >> 3) * (kMpRows * 128) + r * 128 + (((g & 7) ^ (r & 7)) << 4)) =
              o[k];
        }
      }
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
                        const __grid_constant__ CUtensorMap tmap_w, const AttnParams p,
                        const __grid_constant__ FusedParams f) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t tmem = attn_unit<false>(smem, &tmap_kv_score, &tmap_pe, &tmap_qpe, &tmap_kv_value, &tmap_qabs,
                                         &tmap_out, p);
  fused_tail(smem, tmem, &tmap_w, f);
  attn_teardown(tmem);
}

}  // namespace sm100
}  // namespace mla
