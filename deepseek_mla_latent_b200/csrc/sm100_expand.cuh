// sm100_expand.cuh -- the latent KV expansion on tcgen05 for the DeepSeek-V3
// shapes (C = 512, Dn = Dv = 128).
//
// Operation ("Latent KV expansion with split", the operation's description;
// "Naive vs Absorb Attention Implementations in DeepSeek-V3", section "Naive
// Path Execution", is where its output is used):
//   x[t]             = kv_c[t] / sqrt(mean(kv_c[t]^2) + eps) * gamma
//   y[t, h, 0:256]   = x[t] . wkv_b[h*256 : h*256+256]^T
//   K_nope[b,h,s,:]  = y[b*S+s, h, 0:128],  V[b,h,s,:] = y[b*S+s, h, 128:256]
//
// A GEMM of M = tokens, N = 32768, K = 512 that is tensor-bound (512 flop per
// output byte).  Work item = (128-token tile, head): M = 128 tokens, N = 256
// (the head's 128 key rows and 128 value rows of wkv_b), K = 512.  Items are
// ordered tile-major and each CTA (one per SM) takes a contiguous run of them,
// so a CTA keeps its token tile resident and streams the weights of one head
// after another:
//   shared memory: the token tile (128 KB: eight 64-column blocks of 128
//     rows, 128-byte swizzle, one TMA copy), gamma applied in place; a ring of
//     three 32 KB weight stages (64 columns of 256 rows, one TMA copy each).
//   TMEM: two 256-column fp32 accumulators, so the epilogue of one head
//     overlaps the products of the next.
// The RMS factor of a row is a per-row scale of its outputs, applied in the
// epilogue: y = r_t * ((kv_c[t] * gamma) . W^T).
//
// Warps: 0-3 row statistics, gamma and the epilogue (thread = token row =
// TMEM lane), 4 TMA, 5 MMA (one elected lane issues).  Every wait is bounded;
// a wait that runs out raises the device error word and the thread takes its
// exit path.
#pragma once

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kExThreads = 192;
constexpr int kExProducerWarp = 4, kExMmaWarp = 5;
constexpr int kExStages = 3;

struct ExpandSmem {
  static constexpr int kABlock = 128 * 128;                 // 128 rows x 64 columns bf16
  static constexpr int kA = 8 * kABlock;                    // the token tile, 128 KB
  static constexpr int kStage = 256 * 128;                  // 256 weight rows x 64 columns, 32 KB
  static constexpr int kOffStages = kA;
  static constexpr int kOffBars = kOffStages + kExStages * kStage;
  static constexpr int kBytes = kOffBars + 256;
};
constexpr size_t expand_smem_bytes() { return 1024 + ExpandSmem::kBytes; }
static_assert(expand_smem_bytes() <= 232448, "expansion shared memory above the per-CTA limit");

namespace exbar {
constexpr int kBFull = 0, kBEmpty = 3, kAFull = 6, kAReady = 7, kAFree = 8, kAccFull = 9, kAccEmpty = 11, kIdle = 13;
constexpr int kTmemSlot = 31;
}

struct ExpandParams {
  const __nv_bfloat16* gamma;   // [512] or nullptr
  float eps;
  int64_t n_tokens;             // batch * seq_len
  int64_t seq_len;
  int heads;
  int64_t n_items;              // ceil(n_tokens / 128) * heads
  __nv_bfloat16* k_nope;        // [batch, heads, seq_len, 128]
  __nv_bfloat16* v;             // [batch, heads, seq_len, 128]
  int vec32;                    // both outputs 32-byte aligned: whole-sector stores
};

__global__ void __launch_bounds__(kExThreads, 1)
    expand_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const ExpandParams p) {
  using L = ExpandSmem;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  uint64_t* b_full = bars + exbar::kBFull;       // [3] weight stage landed
  uint64_t* b_empty = bars + exbar::kBEmpty;     // [3] weight stage read by the tensor core
  uint64_t* a_full = bars + exbar::kAFull;       // token tile landed
  uint64_t* a_ready = bars + exbar::kAReady;     // gamma applied (128 arrivals)
  uint64_t* a_free = bars + exbar::kAFree;       // the last product reading the tile finished
  uint64_t* acc_full = bars + exbar::kAccFull;   // [2] accumulator holds a finished head
  uint64_t* acc_empty = bars + exbar::kAccEmpty; // [2] accumulator drained (128 arrivals)
  uint64_t* idle = bars + exbar::kIdle;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + exbar::kTmemSlot);
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();

  // this CTA's run of (tile, head) items
  const int64_t i0 = p.n_items * blockIdx.x / gridDim.x, i1 = p.n_items * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kExStages; ++s) {
      ptx::mbar_init(&b_full[s], 1);
      ptx::mbar_init(&b_empty[s], 1);
    }
    ptx::mbar_init(a_full, 1);
    ptx::mbar_init(a_ready, 128);
    ptx::mbar_init(a_free, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&acc_full[s], 1);
      ptx::mbar_init(&acc_empty[s], 128);
    }
    ptx::mbar_init(idle, 1);
    ptx::fence_mbar_init();
  }
  if (warp == kExMmaWarp) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool aligned = (ptx::smem_u32(smem) & 1023u) == 0;   // the swizzled tiles need it
  if (!aligned && threadIdx.x == 0) raise_error(kErrBadSchedule);
  const int64_t run_end = aligned ? i1 : i0;

  if (warp == kExProducerWarp) {
    // ============================================================ TMA
    int a_uses = 0;
    int64_t chunk = 0, prev_tile = -1;
    bool ok = true;
    if (ptx::elect_one()) {
      ptx::prefetch_tmap(&tmap_x);
      ptx::prefetch_tmap(&tmap_w);
    }
    __syncwarp();
    for (int64_t i = i0; ok && i < run_end; ++i) {
      const int64_t tile = i / p.heads;
      const int h = (int)(i % p.heads);
      if (tile != prev_tile) {
        if (a_uses > 0) ok = __all_sync(0xffffffffu, ptx::mbar_wait(a_free, (a_uses - 1) & 1, kErrTimeoutMma));
        if (!ok) break;
        if (ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(a_full, L::kA);
          ptx::tma_load_3d(smem, &tmap_x, a_full, 0, (int32_t)(tile * 128), 0);
        }
        __syncwarp();
        ++a_uses;
        prev_tile = tile;
      }
      for (int kc = 0; kc < 8; ++kc, ++chunk) {
        const int s = (int)(chunk % kExStages);
        const bool w = ptx::mbar_wait(&b_empty[s], (uint32_t)((chunk / kExStages) & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(&b_full[s], L::kStage);
          ptx::tma_load_2d(smem + L::kOffStages + s * L::kStage, &tmap_w, &b_full[s], kc * 64, h * 256);
        }
        __syncwarp();
      }
    }
    // exit path: every copy this CTA started lands before its shared memory goes away
    for (int64_t c = (chunk > kExStages ? chunk - kExStages : 0); c < chunk; ++c)
      ptx::mbar_wait(&b_full[c % kExStages], (uint32_t)((c / kExStages) & 1), kErrTimeoutDrain);
    if (a_uses > 0) ptx::mbar_wait(a_full, (a_uses - 1) & 1, kErrTimeoutDrain);
  } else if (warp == kExMmaWarp) {
    // ============================================================ MMA
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 256, false, false);
    const uint32_t a0 = ptx::smem_u32(smem), b0 = ptx::smem_u32(smem + L::kOffStages);
    int a_uses = 0;
    int64_t chunk = 0, prev_tile = -1, n = 0;
    bool ok = true;
    for (int64_t i = i0; ok && i < run_end; ++i, ++n) {
      const int64_t tile = i / p.heads;
      if (tile != prev_tile) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(a_ready, a_uses & 1, kErrTimeoutSoftmax));
        if (!ok) break;
        ++a_uses;
        prev_tile = tile;
      }
      const int ab = (int)(n & 1);
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&acc_empty[ab], (uint32_t)((n >> 1) & 1) ^ 1, kErrTimeoutMma));
      if (!ok) break;
      ptx::tc_fence_after();
      for (int kc = 0; kc < 8; ++kc, ++chunk) {
        const int s = (int)(chunk % kExStages);
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&b_full[s], (uint32_t)((chunk / kExStages) & 1), kErrTimeoutTmaFull));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t da = ptx::smem_desc(a0 + kc * L::kABlock + ks * 32, 16, 1024, ptx::kSwizzle128);
          const uint64_t db = ptx::smem_desc(b0 + s * L::kStage + ks * 32, 16, 1024, ptx::kSwizzle128);
          if (ptx::elect_one()) ptx::mma_ss(tmem + 256 * ab, da, db, idesc, (kc > 0 || ks > 0) ? 1u : 0u);
          __syncwarp();
        }
        if (ptx::elect_one()) ptx::mma_commit(&b_empty[s]);
        __syncwarp();
      }
      if (!ok) break;
      if (ptx::elect_one()) {
        ptx::mma_commit(&acc_full[ab]);
        if (i + 1 == run_end || (i + 1) / p.heads != tile) ptx::mma_commit(a_free);
      }
      __syncwarp();
    }
    // every product this warp issued has finished before TMEM and shared memory are released
    if (ptx::elect_one()) ptx::mma_commit(idle);
    __syncwarp();
    ptx::mbar_wait(idle, 0, kErrTimeoutDrain);
  } else {
    // ============================================================ warps 0-3
    const uint32_t lane_base = (warp * 32) << 16;
    const int t = (int)(warp * 32 + lane);                // row of the tile = TMEM lane
    int a_uses = 0;
    int64_t prev_tile = -1, n = 0;
    float r = 0.f;
    for (int64_t i = i0; i < run_end; ++i, ++n) {
      const int64_t tile = i / p.heads;
      const int h = (int)(i % p.heads);
      if (tile != prev_tile) {
        bool w = ptx::mbar_wait(a_full, a_uses & 1, kErrTimeoutTmaFull);
        if (!__all_sync(0xffffffffu, w)) break;
        // row t: sum of squares of the raw values; with a gain, x * gamma rewritten in place
        float ss = 0.f;
#pragma unroll 1
        for (int blk = 0; blk < 8; ++blk) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* ptr = reinterpret_cast<uint4*>(smem + blk * L::kABlock + t * 128 + ((c ^ (t & 7)) << 4));
            uint4 x = *ptr;
            uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
              ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
              if (p.gamma) {
                const int col = blk * 64 + c * 8 + 2 * e;
                const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p.gamma + col));
                u[e] = ptx::pack_bf16x2(f.x * g.x, f.y * g.y);
              }
            }
            if (p.gamma) *ptr = make_uint4(u[0], u[1], u[2], u[3]);
          }
        }
        r = rsqrtf(ss * (1.f / 512.f) + p.eps);
        ptx::fence_async_smem();   // the gamma-scaled rows are read by the tensor core
        ptx::mbar_arrive(a_ready);
        ++a_uses;
        prev_tile = tile;
      }
      const int ab = (int)(n & 1);
      bool w = ptx::mbar_wait(&acc_full[ab], (uint32_t)((n >> 1) & 1), kErrTimeoutMma);
      if (!__all_sync(0xffffffffu, w)) break;
      ptx::tc_fence_after();
      const int64_t tok = tile * 128 + t;
      const bool valid = tok < p.n_tokens;
      const int64_t b = valid ? tok / p.seq_len : 0, s = valid ? tok % p.seq_len : 0;
      const int64_t row = ((b * p.heads + h) * p.seq_len + s) * 128;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + lane_base + 256 * ab + 32 * c, v);
        ptx::tmem_wait_ld();
        if (valid) {
          __nv_bfloat16* dst = (c < 4 ? p.k_nope : p.v) + row + 32 * (c & 3);
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q)
            pk[q] = ptx::pack_bf16x2(__uint_as_float(v[2 * q]) * r, __uint_as_float(v[2 * q + 1]) * r);
          if (p.vec32) {
            // a lane's row is 256 bytes: 32-byte stores fill whole L2 sectors (16-byte stores from
            // lanes 256 bytes apart would each write half a sector)
            ptx::st_global_v8(dst, *reinterpret_cast<const uint32_t(*)[8]>(&pk[0]));
            ptx::st_global_v8(dst + 16, *reinterpret_cast<const uint32_t(*)[8]>(&pk[8]));
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int q = 0; q < 4; ++q) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&acc_empty[ab]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kExMmaWarp) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace sm100
}  // namespace mla
