// sm100_fmha.cuh -- per-head attention over materialised keys and values on
// tcgen05: the naive path of DeepSeek-V3 multi-head latent attention for a
// chunked prefill.
//
// Operation ("Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Naive Path Execution"): with the per-head keys and values already
// expanded from the latent cache ("Latent KV expansion with split": K_nope and
// V per head, the rotary key shared by every head), for query row i of a
// sequence and head h
//   S[i,j] = (q_nope[i,h,:] . K_nope[h,j,:] + q_pe[i,h,:] . pe[j,:]) * scale
//   P      = softmax_j(S)   (query i of s new queries over t keys sees j <= t - s + i)
//   out[i,h,:] = sum_j P[i,j] V[h,j,:]
// The head dimension of the scores is Dn + R = 192 and of the values Dv = 128;
// the result is already the attention output (no latent output projection).
//
// One CTA per SM, persistent over work units (sequence, head, pair of 128-row
// query tiles A and B).  The two query tiles (128 rows x 192 columns each,
// three 64-column blocks, 128-byte swizzle) stay in shared memory for the
// unit and share one stream of key tiles (128 keys x 192: two K_nope blocks
// and the rotary block, one stage) and value tiles (128 keys x 128, two
// stages): every key and value tile serves both query tiles.  TMEM per query
// tile x: S at 256x (128 columns; P, bf16 pairs, overwrites its first 64
// columns) and O at 256x + 128.  Warps 0-3 run the softmax and epilogue of
// tile A, warps 4-7 those of tile B (thread = query row = TMEM lane), warp 8
// loads (TMA), warp 9 issues the MMAs in the order QK_A(j+1) after PV_A(j),
// QK_B(j+1) after PV_B(j): while one warpgroup computes the exponentials of
// its tile, the tensor core runs the other tile's products.  The commit that
// signals S_x(j) also covers PV_x(j-1) (issued before it), so when a
// warpgroup sees its scores, O_x already holds every earlier product and may
// be rescaled in place.  The reference max of a row moves lazily (only when a
// tile's max exceeds it by more than 2^8), so O is rescaled rarely; P <= 2^8.
// Every wait is bounded; a wait that runs out raises the device error word
// and the thread takes its exit path.
#pragma once

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kFaThreads = 320;
constexpr int kFaProducerWarp = 8, kFaMmaWarp = 9;
constexpr int kFaTile = 128;                 // query rows per tile, keys per tile
constexpr float kFaRescale = 8.0f;           // log2 units

struct FaLayout {
  static constexpr int kBlock = 128 * 128;                  // 128 rows x 64 columns bf16
  static constexpr int kQ = 3 * kBlock;                     // query tile: nope 0..127, rotary 128..191
  static constexpr int kK = 3 * kBlock;                     // key tile: K_nope blocks 0, 1, rotary block
  static constexpr int kV = 2 * kBlock;                     // value tile
  static constexpr int kVStages = 2;
  static constexpr int kOffQ = 0;                           // query tiles A, B
  static constexpr int kOffK = kOffQ + 2 * kQ;              // one key stage
  static constexpr int kOffV = kOffK + kK;                  // two value stages
  static constexpr int kOffBars = kOffV + kVStages * kV;
  static constexpr int kBytes = kOffBars + 256;
};
constexpr size_t fa_smem_bytes() { return 1024 + FaLayout::kBytes; }
static_assert(fa_smem_bytes() <= 232448, "attention shared memory above the per-CTA limit");

namespace fabar {
// [2]: one per query tile (A, B) or per value stage
constexpr int kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = 3, kVFull = 4, kVEmpty = 6, kSFull = 8, kPFull = 10,
              kODone = 12, kOFree = 14, kIdle = 16;
constexpr int kTmemSlot = 31;
}  // namespace fabar

// TMEM of query tile x: S (and P over its first 64 columns) at kFaColTile * x, O at kFaColTile * x + kFaColO.
constexpr uint32_t kFaColTile = 256, kFaColO = 128;

struct FaParams {
  const int* cu_q;        // [batch + 1]
  const int* cu_k;        // [batch + 1]
  int batch;
  int heads;
  int q_pairs;            // pairs of query tiles per sequence (ceil(max_seqlen_q / 256))
  int64_t n_units;        // batch * heads * q_pairs
  int64_t n_q;            // query rows
  int64_t kv_rows;
  float scale_log2;       // softmax_scale * log2(e)
  __nv_bfloat16* out;     // [n_q, heads, 128]
};

// A unit's sequence, head and pair of query tiles, its first query row and first key row, the
// sequence's query and key counts, the query rows of tiles A and B, and the keys the pair needs
// (nk tiles).
struct FaUnit {
  int b, h, qp;
  int64_t q0, k0, s, t, kend;
  int64_t rows[2];
  int nk;
};

__device__ __forceinline__ float fa_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ FaUnit fa_unit(const FaParams& p, int64_t u) {
  FaUnit x;
  x.qp = (int)(u % p.q_pairs);
  x.h = (int)((u / p.q_pairs) % p.heads);
  x.b = (int)(u / ((int64_t)p.q_pairs * p.heads));
  const int64_t qa = __ldg(p.cu_q + x.b), qb = __ldg(p.cu_q + x.b + 1);
  x.s = max64(0, min64(qb, p.n_q) - max64(0, qa));
  x.q0 = max64(0, qa) + (int64_t)x.qp * 2 * kFaTile;
  const int64_t ka = min64(max64(0, __ldg(p.cu_k + x.b)), p.kv_rows);
  x.k0 = ka;
  x.t = max64(0, min64((int64_t)__ldg(p.cu_k + x.b + 1), p.kv_rows) - ka);
  const int64_t r0 = x.s - (int64_t)x.qp * 2 * kFaTile;   // query rows from tile A on
  x.rows[0] = max64(0, min64(kFaTile, r0));
  x.rows[1] = max64(0, min64(kFaTile, r0 - kFaTile));
  if (x.rows[0] <= 0) {
    x.kend = 0;
    x.nk = 0;
    return x;
  }
  // the pair's last row sees keys 0 .. t - s + (its index)
  x.kend = min64(x.t, max64(0, x.t - x.s + (int64_t)x.qp * 2 * kFaTile + x.rows[0] + x.rows[1]));
  x.nk = (int)((x.kend + kFaTile - 1) / kFaTile);
  return x;
}

__global__ void __launch_bounds__(kFaThreads, 1)
    fmha_kernel(const __grid_constant__ CUtensorMap tmap_q,      // q [n_q, H, 192] viewed 3-D
                const __grid_constant__ CUtensorMap tmap_knope,  // K_nope [H, kv_rows, 128] viewed 3-D
                const __grid_constant__ CUtensorMap tmap_pe,     // pe [kv_rows, 64]
                const __grid_constant__ CUtensorMap tmap_v,      // V [H, kv_rows, 128] viewed 3-D
                const FaParams p) {
  using L = FaLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  uint64_t* q_full = bars + fabar::kQFull;     // both query tiles landed
  uint64_t* q_empty = bars + fabar::kQEmpty;   // the unit's last score product finished
  uint64_t* k_full = bars + fabar::kKFull;     // key tile landed
  uint64_t* k_empty = bars + fabar::kKEmpty;   // both score products of the key tile finished
  uint64_t* v_full = bars + fabar::kVFull;     // [2] value tile landed
  uint64_t* v_empty = bars + fabar::kVEmpty;   // [2] both value products of the tile finished
  uint64_t* s_full = bars + fabar::kSFull;     // [2] score product of tile x committed (and every product before)
  uint64_t* p_full = bars + fabar::kPFull;     // [2] P of tile x written, O_x rescaled (128 arrivals)
  uint64_t* o_done = bars + fabar::kODone;     // [2] the unit's last value product of tile x finished
  uint64_t* o_free = bars + fabar::kOFree;     // [2] the epilogue of tile x read O_x (128 arrivals)
  uint64_t* idle = bars + fabar::kIdle;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + fabar::kTmemSlot);
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_empty, 1);
    ptx::mbar_init(k_full, 1);
    ptx::mbar_init(k_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&v_full[i], 1);
      ptx::mbar_init(&v_empty[i], 1);
      ptx::mbar_init(&s_full[i], 1);
      ptx::mbar_init(&p_full[i], 128);
      ptx::mbar_init(&o_done[i], 1);
      ptx::mbar_init(&o_free[i], 128);
    }
    ptx::mbar_init(idle, 1);
    ptx::fence_mbar_init();
  }
  if (warp == kFaMmaWarp) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  ptx::griddep_wait();

  if (warp == kFaProducerWarp) {
    // ============================================================ producer
    if (ptx::elect_one()) {
      ptx::prefetch_tmap(&tmap_q);
      ptx::prefetch_tmap(&tmap_knope);
      ptx::prefetch_tmap(&tmap_pe);
      ptx::prefetch_tmap(&tmap_v);
    }
    __syncwarp();
    int64_t kc = 0, vc = 0;   // key / value tiles issued by this CTA
    int units = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; ok && u < p.n_units; u += gridDim.x) {
      const FaUnit x = fa_unit(p, u);
      if (x.nk == 0) continue;
      // both query tiles (the previous unit's score products must have finished)
      bool w = units == 0 || ptx::mbar_wait(q_empty, (units - 1) & 1, kErrTimeoutStageFree);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      if (ptx::elect_one()) {
        ptx::mbar_arrive_expect_tx(q_full, 2 * L::kQ);
        for (int t = 0; t < 2; ++t)
          for (int blk = 0; blk < 3; ++blk)
            ptx::tma_load_3d(smem + L::kOffQ + t * L::kQ + blk * L::kBlock, &tmap_q, q_full, 64 * blk, x.h,
                             (int)(x.q0 + t * kFaTile));
      }
      __syncwarp();
      ++units;
      // key tile j once both score products of tile j-1 finished, then value tile j into its stage
      for (int j = 0; j < x.nk && ok; ++j) {
        const int row = (int)(x.k0 + (int64_t)j * kFaTile);
        w = ptx::mbar_wait(k_empty, (int)(kc & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (ptx::elect_one()) {
          uint8_t* dst = smem + L::kOffK;
          ptx::mbar_arrive_expect_tx(k_full, L::kK);
          ptx::tma_load_3d(dst, &tmap_knope, k_full, 0, row, x.h);
          ptx::tma_load_3d(dst + L::kBlock, &tmap_knope, k_full, 64, row, x.h);
          ptx::tma_load_2d(dst + 2 * L::kBlock, &tmap_pe, k_full, 0, row);
        }
        __syncwarp();
        ++kc;
        const int st = (int)(vc % L::kVStages);
        w = ptx::mbar_wait(&v_empty[st], (int)((vc / L::kVStages) & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (ptx::elect_one()) {
          uint8_t* dst = smem + L::kOffV + st * L::kV;
          ptx::mbar_arrive_expect_tx(&v_full[st], L::kV);
          ptx::tma_load_3d(dst, &tmap_v, &v_full[st], 0, row, x.h);
          ptx::tma_load_3d(dst + L::kBlock, &tmap_v, &v_full[st], 64, row, x.h);
        }
        __syncwarp();
        ++vc;
      }
    }
    // exit path: every copy this CTA started has landed before its shared memory goes away
    if (kc > 0) ptx::mbar_wait(k_full, (int)((kc - 1) & 1), kErrTimeoutDrain);
    for (int64_t i = (vc > L::kVStages ? vc - L::kVStages : 0); i < vc; ++i)
      ptx::mbar_wait(&v_full[i % L::kVStages], (int)((i / L::kVStages) & 1), kErrTimeoutDrain);
    if (units > 0) ptx::mbar_wait(q_full, (units - 1) & 1, kErrTimeoutDrain);
    __syncwarp();
  } else if (warp == kFaMmaWarp) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, kFaTile, false, false);
    constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(128, 128, false, true);
    const uint64_t d_smem = ptx::smem_desc(ptx::smem_u32(smem), 16, 1024, ptx::kSwizzle128);
    const uint64_t d_v = ptx::smem_desc(ptx::smem_u32(smem), L::kBlock, 1024, ptx::kSwizzle128);
    int64_t kc = 0, vc = 0;   // key / value tiles consumed
    int64_t tcx[2] = {0, 0};  // score tiles of query tile x (S / P uses)
    int units = 0;
    bool ok = true;
    // S_x = Q_x K^T over the 192 columns (12 products), then its commit
    auto qk = [&](int xt) {
      ptx::tc_fence_after();
      const uint64_t dq = d_smem + (uint32_t)((L::kOffQ + xt * L::kQ) >> 4);
      const uint64_t dk = d_smem + (uint32_t)(L::kOffK >> 4);
#pragma unroll
      for (int blk = 0; blk < 3; ++blk)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t off = (uint32_t)((blk * L::kBlock + ks * 32) >> 4);
          if (ptx::elect_one())
            ptx::mma_ss(tmem + kFaColTile * xt, dq + off, dk + off, idesc_s, (blk > 0 || ks > 0) ? 1u : 0u);
          __syncwarp();
        }
      if (ptx::elect_one()) ptx::mma_commit(&s_full[xt]);
      __syncwarp();
    };
    // O_x (+)= P_x V over the tile's 128 keys (8 products, A = P from TMEM)
    auto pv = [&](int xt, int vs, bool first) {
      ptx::tc_fence_after();
      const uint64_t db = d_v + (uint32_t)((L::kOffV + vs * L::kV) >> 4);
#pragma unroll
      for (int ks = 0; ks < kFaTile / 16; ++ks) {
        if (ptx::elect_one())
          ptx::mma_ts(tmem + kFaColTile * xt + kFaColO, tmem + kFaColTile * xt + 8 * ks,
                      db + (uint32_t)((ks * 2048) >> 4), idesc_o, (first && ks == 0) ? 0u : 1u);
        __syncwarp();
      }
    };
    for (int64_t u = blockIdx.x; ok && u < p.n_units; u += gridDim.x) {
      const FaUnit x = fa_unit(p, u);
      if (x.nk == 0) continue;
      bool w = ptx::mbar_wait(q_full, units & 1, kErrTimeoutTmaFull) &&
               ptx::mbar_wait(k_full, (int)(kc & 1), kErrTimeoutTmaFull);
      if (!__all_sync(0xffffffffu, w)) break;
      // the score products of key tile 0 for both query tiles
      qk(0);
      qk(1);
      if (ptx::elect_one()) {
        ptx::mma_commit(k_empty);
        if (x.nk == 1) ptx::mma_commit(q_empty);
      }
      __syncwarp();
      ++kc;
      for (int j = 0; ok && j < x.nk; ++j) {
        const int vs = (int)(vc % L::kVStages);
        w = ptx::mbar_wait(&v_full[vs], (int)((vc / L::kVStages) & 1), kErrTimeoutTmaFull);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
#pragma unroll 1
        for (int xt = 0; xt < 2; ++xt) {
          // P_x(j) written; for the unit's first product O_x must have been read out
          w = ptx::mbar_wait(&p_full[xt], (int)(tcx[xt] & 1), kErrTimeoutSoftmax);
          if (j == 0 && units > 0) w = w && ptx::mbar_wait(&o_free[xt], (units - 1) & 1, kErrTimeoutSoftmax);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          pv(xt, vs, j == 0);
          ++tcx[xt];
          if (ptx::elect_one()) {
            if (xt == 1) ptx::mma_commit(&v_empty[vs]);
            if (j == x.nk - 1) ptx::mma_commit(&o_done[xt]);
          }
          __syncwarp();
          // the score product of key tile j+1 (it overwrites P_x(j), which the value product above
          // reads first: products issued by one thread run in order)
          if (j + 1 < x.nk) {
            if (xt == 0) {
              w = ptx::mbar_wait(k_full, (int)(kc & 1), kErrTimeoutTmaFull);
              if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            }
            qk(xt);
            if (xt == 1) {
              if (ptx::elect_one()) {
                ptx::mma_commit(k_empty);
                if (j + 1 == x.nk - 1) ptx::mma_commit(q_empty);
              }
              __syncwarp();
              ++kc;
            }
          }
        }
        ++vc;
      }
      ++units;
    }
    // nothing of ours may still run in the tensor core when TMEM is freed
    if (ptx::elect_one()) ptx::mma_commit(idle);
    __syncwarp();
    ptx::mbar_wait(idle, 0, kErrTimeoutDrain);
    __syncwarp();
  } else {
    // ============================================================ softmax + epilogue of query tile xt
    const int xt = (int)(warp >> 2);
    const int r = (int)((warp & 3) * 32 + lane);       // query row within the tile = TMEM lane
    const uint32_t t_s = tmem + ((uint32_t)((warp & 3) * 32) << 16) + kFaColTile * xt;
    const uint32_t t_o = t_s + kFaColO;
    const float sl2 = p.scale_log2;
    int64_t tc = 0;
    int units = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; ok && u < p.n_units; u += gridDim.x) {
      const FaUnit x = fa_unit(p, u);
      const int64_t i_row = (int64_t)x.qp * 2 * kFaTile + (int64_t)xt * kFaTile + r;   // index in the sequence
      const bool row_valid = i_row < x.s;
      if (x.nk == 0) {
        // query rows that see no key get zeros
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((x.q0 + xt * kFaTile + r) * p.heads + x.h) * 128);
          for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      // keys this row sees: 0 .. t - s + i_row; rows past the sequence's queries are computed
      // over the pair's keys and never stored
      const int64_t lim = row_valid ? min64(x.t, max64(0, x.t - x.s + i_row + 1)) : x.kend;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < x.nk; ++j) {
        bool w = ptx::mbar_wait(&s_full[xt], (int)(tc & 1), kErrTimeoutMma);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t a[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(t_s + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&a[32 * c]));
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::reg_fence32(&a[32 * c]);
        const int n_valid = (int)max64(0, min64(kFaTile, lim - (int64_t)j * kFaTile));   // this row's keys in the tile
        float mx = -INFINITY;
        if (n_valid >= kFaTile) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 128; ++i) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(a[i]));
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        } else {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i < n_valid) mx = fmaxf(mx, __uint_as_float(a[i]));
        }
        mx *= sl2;
        const float m_new = (mx > m_ref + kFaRescale) ? mx : m_ref;
        const float f = (m_ref == -INFINITY || m_new == m_ref) ? 1.f : fa_exp2(m_ref - m_new);
        // O_x holds the value products of tiles < j (the commit of S_x(j) covers them): rescale
        // it in place when the reference moved
        if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(t_o + 32 * c, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            ptx::tmem_st32(t_o + 32 * c, o);
          }
        }
        if (m_new != m_ref) {
          l *= f;
          m_ref = m_new;
        }
        // P = 2^(s * scale * log2(e) - m) as bf16 pairs over S's first 64 columns, 32 columns (64
        // keys) at a time; keys the row does not see weigh exactly 0
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
          if (n_valid >= kFaTile) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float e0 = fa_exp2(fmaf(__uint_as_float(a[64 * hf + 2 * i]), sl2, -m_new));
              const float e1 = fa_exp2(fmaf(__uint_as_float(a[64 * hf + 2 * i + 1]), sl2, -m_new));
              ls0 += e0;
              ls1 += e1;
              pk[i] = ptx::pack_bf16x2(e0, e1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int k = 64 * hf + 2 * i;
              const float e0 = k < n_valid ? fa_exp2(fmaf(__uint_as_float(a[k]), sl2, -m_new)) : 0.f;
              const float e1 = k + 1 < n_valid ? fa_exp2(fmaf(__uint_as_float(a[k + 1]), sl2, -m_new)) : 0.f;
              ls0 += e0;
              ls1 += e1;
              pk[i] = ptx::pack_bf16x2(e0, e1);
            }
          }
          ptx::tmem_st32(t_s + 32 * hf, pk);
        }
        l += ls0 + ls1;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_full[xt]);
        ++tc;
      }
      if (!ok) break;
      // epilogue: O / l as bf16 into out[row, h, :]; then O_x may be overwritten
      bool w = ptx::mbar_wait(&o_done[xt], units & 1, kErrTimeoutMma);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = p.out + ((x.q0 + xt * kFaTile + r) * p.heads + x.h) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        ptx::tmem_ld32(t_o + 32 * c, o);
        ptx::tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            reinterpret_cast<uint4*>(dst + 32 * c)[v] =
                make_uint4(ptx::pack_bf16x2(__uint_as_float(o[8 * v]) * inv, __uint_as_float(o[8 * v + 1]) * inv),
                           ptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv),
                           ptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv),
                           ptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv));
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&o_free[xt]);
      ++units;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kFaMmaWarp) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace sm100
}  // namespace mla
