// sm100_proj.cuh -- the two per-head projections of the absorb path as
// tcgen05 GEMMs ("Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Absorb Path Execution": the einsum folding q_nope through the key
// rows of wkv_b, and the final einsum with its value rows).
//
// Both are computed "weight as the M operand": for head h
//   absorb:  q_abs[n,h,c] = sum_d W_k[h][d][c] q[n,h,d]   M = c (128-row tiles), K = d (128)
//   out:     out[n,h,d]   = sum_c W_v[h][d][c] o[n,h,c]   M = d (128),          K = c (512)
// with the query rows n as the N operand (16..256 per tile).  At decode
// sizes (n = batch) the weight read is the whole cost, so M on the weight
// keeps each weight byte read once per call whatever the batch.
//
// One CTA per (M tile, head, N tile), four warps: warp 0 feeds a
// STAGES-deep ring of 64-wide K chunks with TMA, warp 1 issues the MMAs into
// a TMEM accumulator (128 lanes x N columns fp32) -- both loop with the whole
// warp and issue from one elected lane -- then all four warps drain TMEM
// (warp w owns lanes 32w..32w+31) and store bf16.
#pragma once

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kProjThreads = 128;
constexpr int kProjBoxK = 64;   // K elements per chunk = one 128-byte swizzle row

template <int N_TILE>
struct ProjSmem {
  static constexpr int kA = 128 * kProjBoxK * 2;                              // 16 KB per stage
  static constexpr int kB = ((N_TILE * kProjBoxK * 2 + 1023) / 1024) * 1024;  // N_TILE rows of 128 B
  static constexpr int kStage = kA + kB;
};

// A_MN: A (the weight) is stored with M contiguous (absorb: W_k[h][d][c], M = c).
template <bool A_MN, int N_TILE, int STAGES>
__global__ void __launch_bounds__(kProjThreads, 1) proj_kernel(
    const __grid_constant__ CUtensorMap tmap_w,   // wkv_b [H*(Dn+Dv), C] bf16, 2D
    const __grid_constant__ CUtensorMap tmap_x,   // activations [N, H, K] bf16, 3D (row stride free)
    int k_chunks, int w_row_base, int w_rows_per_head, int n_rows, __nv_bfloat16* __restrict__ out,
    int64_t out_row_stride, int out_head_stride) {
  using L = ProjSmem<N_TILE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStage);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int m_tile = blockIdx.x, h = blockIdx.y, n_tile = blockIdx.z;
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();
  constexpr uint32_t kTmemCols = N_TILE <= 32 ? 32 : (N_TILE <= 64 ? 64 : (N_TILE <= 128 ? 128 : 256));

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  // weight chunk i into stage s; the stage's barrier expects the weight and the activation bytes
  auto load_w = [&](int i, int s) {
    uint8_t* a = smem + s * L::kStage;
    ptx::mbar_arrive_expect_tx(&full[s], L::kA + N_TILE * kProjBoxK * 2);
    if (A_MN) {
      // two 64(c) x 64(d) boxes: M elements 0..63 and 64..127 of this tile
      const int c0 = m_tile * 128, row = w_row_base + h * w_rows_per_head + i * kProjBoxK;
      ptx::tma_load_2d(a, &tmap_w, &full[s], c0, row);
      ptx::tma_load_2d(a + L::kA / 2, &tmap_w, &full[s], c0 + 64, row);
    } else {
      // one 64(c) x 128(d) box: K elements i*64.., all 128 M rows
      ptx::tma_load_2d(a, &tmap_w, &full[s], i * kProjBoxK, w_row_base + h * w_rows_per_head);
    }
  };
  // The weights are never written by the kernels that may run before this one in the stream, so
  // the first stages' weight copies start before the dependency wait and overlap the previous
  // kernel's tail; the activations (the previous kernel's output) are read only after it.
  const int early = warp == 0 ? (k_chunks < STAGES ? k_chunks : STAGES) : 0;
  if (warp == 0) {
    if (ptx::elect_one())
      for (int i = 0; i < early; ++i) load_w(i, i);
    __syncwarp();
  }
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  int issued = 0;  // chunks whose TMA the producer started
  if (warp == 0) {
    // producer: the whole warp loops, one elected lane issues
    for (int i = 0; i < k_chunks; ++i) {
      const int s = i % STAGES;
      if (i >= early) {
        const bool w = ptx::mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) break;
        if (ptx::elect_one()) load_w(i, s);
        __syncwarp();
      }
      if (ptx::elect_one())
        ptx::tma_load_3d(smem + s * L::kStage + L::kA, &tmap_x, &full[s], i * kProjBoxK, h, n_tile * N_TILE);
      __syncwarp();
      issued = i + 1;
    }
  } else if (warp == 1) {
    // MMA issuer: the whole warp loops, one elected lane issues
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, N_TILE, A_MN, false);
    for (int i = 0; i < k_chunks; ++i) {
      const int s = i % STAGES;
      const bool w = ptx::mbar_wait(&full[s], (i / STAGES) & 1, kErrTimeoutTmaFull);
      if (!__all_sync(0xffffffffu, w)) break;
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + s * L::kStage);
      const uint32_t b = a + L::kA;
#pragma unroll
      for (int ks = 0; ks < kProjBoxK / 16; ++ks) {
        const uint64_t da = A_MN ? ptx::smem_desc(a + ks * 2048, L::kA / 2, 1024, ptx::kSwizzle128)
                                 : ptx::smem_desc(a + ks * 32, 16, 1024, ptx::kSwizzle128);
        const uint64_t db = ptx::smem_desc(b + ks * 32, 16, 1024, ptx::kSwizzle128);
        if (ptx::elect_one()) ptx::mma_ss(tmem_d, da, db, idesc, (i > 0 || ks > 0) ? 1u : 0u);
        __syncwarp();
      }
      if (ptx::elect_one()) ptx::mma_commit(&empty[s]);
      __syncwarp();
    }
    if (ptx::elect_one()) ptx::mma_commit(done);
    __syncwarp();
  }

  // Epilogue: TMEM -> registers -> bf16 -> global.
  const bool ok = ptx::mbar_wait(done, 0, kErrTimeoutMma);
  ptx::tc_fence_after();
  if (ok) {
    const int m = warp * 32 + lane;
    __nv_bfloat16* o = out + (int64_t)h * out_head_stride + m_tile * 128 + m;
    const int n_base = n_tile * N_TILE;
#pragma unroll 1
    for (int n0 = 0; n0 < N_TILE; n0 += 16) {
      if (n_base + n0 >= n_rows) break;   // warp-uniform
      uint32_t r[16];
      ptx::tmem_ld16(tmem_d + ((warp * 32) << 16) + n0, r);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n_base + n0 + j;
        if (n < n_rows) o[(int64_t)n * out_row_stride] = __float2bfloat16_rn(__uint_as_float(r[j]));
      }
    }
  }
  // Exit path: let every TMA this CTA started land before the CTA's shared memory is released.
  if (warp == 0) {
    for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
      ptx::mbar_wait(&full[i % STAGES], (i / STAGES) & 1, kErrTimeoutDrain);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem_d, kTmemCols);
}

template <int N_TILE, int STAGES>
constexpr size_t proj_smem_bytes() {
  return 1024 + STAGES * ProjSmem<N_TILE>::kStage + (2 * STAGES + 1) * 8 + 16;
}

}  // namespace sm100
}  // namespace mla
