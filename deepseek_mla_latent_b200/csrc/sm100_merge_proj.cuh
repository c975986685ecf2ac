// sm100_merge_proj.cuh -- the split merge fused into the output projection of
// a decode step ("Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Absorb Path Execution": the last einsum, out = o_lat . W_v^T, with
// o_lat the log-sum-exp merge of the attention call's split partials).
//
// One CTA per (head h, 16 query rows), 512 threads:
//   * before the dependency wait, warp 0 starts the TMA copies of W_v[h]
//     (128 value rows x 512 columns, eight 16 KB K chunks): the weights are
//     not written by the attention kernel, which has already pulled them into
//     L2 by the time this kernel can run;
//   * after it, each warp computes the merge weights of two rows (the same
//     warp-collective code as merge_splits_kernel), then every thread merges
//     (row, 8-column) items of the bf16 partials in split order into o_lat,
//     rounds to bf16 and writes them as the B operand (16 rows x 64 columns per
//     K chunk, K-major, 128-byte swizzle) -- so o_lat never goes to memory;
//   * warp 1 issues the 32 tcgen05.mma (M = 128 value rows, N = 16, K = 16)
//     into TMEM; warps 0-3 store out[n, h, :] from TMEM.
// The merge arithmetic and the product are those of merge_splits_kernel
// followed by proj_kernel (same order of operations), so the results match
// that pair of kernels bit for bit.
#pragma once

#include "sm100_attn.cuh"

namespace mla {
namespace sm100 {

constexpr int kMergeProjThreads = 512;
constexpr int kMpRows = 16;            // query rows per CTA = the MMA's N
constexpr int kMpMaxSplits = 256;

struct MergeProjSmem {
  static constexpr int kW = 128 * 128;                      // one K chunk of W_v[h]: 128 rows x 64 columns
  static constexpr int kChunks = 8;
  static constexpr int kOffB = kChunks * kW;                // B: 8 K chunks x 16 rows x 128 B
  static constexpr int kB = kMpRows * 128;
  static constexpr int kOffWt = kOffB + kChunks * kB;       // merge weight of (split, row): [256][16] floats
  static constexpr int kOffInv = kOffWt + kMpMaxSplits * kMpRows * 4;   // 1 / row sum [16]
  static constexpr int kOffBars = kOffInv + kMpRows * 4;
  static constexpr int kBytes = kOffBars + 128;
};

__global__ void __launch_bounds__(kMergeProjThreads, 1)
    merge_proj_kernel(const __grid_constant__ CUtensorMap tmap_w,   // wkv_b [H*256, 512], boxes 64 x 128
                      const __nv_bfloat16* __restrict__ part_o, const float* __restrict__ part_ml, int num_splits,
                      int n_q, int heads, __nv_bfloat16* __restrict__ out) {
  using L = MergeProjSmem;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + L::kOffBars);   // [8] K chunk of W landed
  uint64_t* done = wfull + L::kChunks;                                  // the products finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* wt = reinterpret_cast<float*>(smem + L::kOffWt);
  float* inv_s = reinterpret_cast<float*>(smem + L::kOffInv);
  const int h = blockIdx.x, n0 = blockIdx.y * kMpRows;
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&tmap_w);
    for (int k = 0; k < L::kChunks; ++k) ptx::mbar_init(&wfull[k], 1);
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, 32);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0) {
    if (ptx::elect_one()) {
      // all eight K chunks of W_v[h] in one copy (the map's third axis steps through them)
      ptx::mbar_arrive_expect_tx(&wfull[0], L::kChunks * L::kW);
      ptx::tma_load_3d(smem, &tmap_w, &wfull[0], 0, h * 256 + 128, 0);
    }
    __syncwarp();
  }
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  // merge weights: warp w handles row w
  const int64_t split_stride = (int64_t)n_q * heads;
  for (int r = (int)warp; r < kMpRows; r += kMergeProjThreads / 32) {
    const int64_t n = n0 + r;
    if (n >= n_q) continue;   // warp-uniform
    const float2* ml = reinterpret_cast<const float2*>(part_ml) + n * heads + h;
    float M, inv;
    const float w_lane = merge_weights(ml, split_stride, num_splits, (int)lane, M, inv);
    for (int s = (int)lane; s < num_splits; s += 32) {
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

  // merge (row r, 16-byte column group g) items into the B operand, one per thread at a time
  // with the loads of up to kInFlight splits in flight together
  const int64_t step = split_stride * 512 / 8;   // one split further, in 16-byte units
  constexpr int kInFlight = 16;
  for (int it = (int)threadIdx.x; it < kMpRows * 64; it += kMergeProjThreads) {
    const int r = it >> 6, g = it & 63;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (n0 + r < n_q) {   // warp-uniform (a warp covers 32 columns of one row)
      const uint4* src = reinterpret_cast<const uint4*>(part_o + (((int64_t)n0 + r) * heads + h) * 512) + g;
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = 0.f;
      for (int s0 = 0; s0 < num_splits; s0 += kInFlight) {
        uint4 v[kInFlight];
#pragma unroll
        for (int s = 0; s < kInFlight; ++s)
          if (s0 + s < num_splits) v[s] = __ldcg(src + (s0 + s) * step);
#pragma unroll
        for (int s = 0; s < kInFlight; ++s)
          if (s0 + s < num_splits) {
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
    // K chunk g/8, row r, 16-byte column g%8 of that chunk (K-major, 128-byte swizzle)
    *reinterpret_cast<uint4*>(smem + L::kOffB + (g >> 3) * L::kB + r * 128 + (((g & 7) ^ (r & 7)) << 4)) = o;
  }
  ptx::fence_async_smem();
  __syncthreads();

  if (warp == 1) {
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kMpRows, false, false);
    bool ok = true;
    for (int k = 0; ok && k < L::kChunks; ++k) {
      if (k == 0) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&wfull[0], 0, kErrTimeoutTmaFull));
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + k * L::kW), b = ptx::smem_u32(smem + L::kOffB + k * L::kB);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ptx::elect_one())
          ptx::mma_ss(tmem, ptx::smem_desc(a + ks * 32, 16, 1024, ptx::kSwizzle128),
                      ptx::smem_desc(b + ks * 32, 16, 1024, ptx::kSwizzle128), idesc, (k | ks) ? 1u : 0u);
        __syncwarp();
      }
    }
    if (ptx::elect_one()) ptx::mma_commit(done);
    __syncwarp();
  }
  if (warp < 4) {
    // out[n, h, d]: TMEM lane d (value row), column n - n0
    const bool ok = ptx::mbar_wait(done, 0, kErrTimeoutMma);
    ptx::tc_fence_after();
    if (ok) {
      uint32_t rr[16];
      ptx::tmem_ld16(tmem + ((warp * 32) << 16), rr);
      ptx::tmem_wait_ld();
      const int d = (int)(warp * 32 + lane);
#pragma unroll
      for (int j = 0; j < kMpRows; ++j) {
        const int64_t n = n0 + j;
        if (n < n_q) out[(n * heads + h) * 128 + d] = __float2bfloat16_rn(__uint_as_float(rr[j]));
      }
    }
  }
  // every weight copy has landed before the shared memory goes away
  if (warp == 0)
    ptx::mbar_wait(&wfull[0], 0, kErrTimeoutDrain);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 32);
}

constexpr size_t merge_proj_smem_bytes() { return 1024 + MergeProjSmem::kBytes; }

}  // namespace sm100
}  // namespace mla
