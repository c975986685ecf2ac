// sm100_attn.cuh -- latent attention on tcgen05 for the DeepSeek-V3 shapes
// (C = 512 latent columns, R = 64 rotary columns, 128 heads per row block).
//
// Operation ("Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Absorb Path Execution"): for one query row and 128 heads
//   S[h,t] = (q_abs[h,:] . kv[t,:] + q_pe[h,:] . pe[t,:]) * scale
//   P      = softmax_t(S)   (keys past the row's visible limit masked)
//   o[h,:] = sum_t P[h,t] kv[t,:]
// The latent cache serves as both key and value, so one shared-memory tile
// of kv feeds both products: K-major for S = Q K^T, MN-major for O = P V.
//
// Why a CTA pair: the fp32 accumulator O for 128 heads x 512 columns is
// 256 KB, all of one SM's tensor memory, leaving nothing for S.  So the two
// CTAs of a cluster split the latent columns: CTA r keeps O[:, 256r..256r+255]
// in TMEM and loads only those kv columns (plus rotary columns 32r..32r+31),
// so no cache byte is read twice.  Each CTA computes the partial score over
// its 288 contraction columns; the two partials (rounded to fp16 on both
// sides, so both CTAs add the same two numbers) are exchanged through
// distributed shared memory with st.async, summed, and both CTAs run the
// same softmax, getting bit-identical P.
//
// Tensor memory (512 columns x 128 lanes, lane = head):
//   [  0,256) O accumulator (fp32)       [256,384) this CTA's half of q_abs (bf16 pairs, MMA A operand)
//   [384,448) S buffer 0 (fp32)          [448,512) S buffer 1
// Shared memory: a 4-stage ring of 64-key tiles (4 x 8 KB latent boxes with
// 128-byte swizzle + 4 KB rotary box with 64-byte swizzle), this CTA's q_pe
// half (128 x 32), the P buffer (128 heads x 64 keys bf16, the A operand of
// O += P V), a one-slot outbox and a two-slot inbox of fp16 partial scores
// (one 16 KB bulk copy per tile).  P lives in shared memory so an S buffer is
// free as soon as the softmax has read it: QK of tile j+2 does not wait for
// the P V product of tile j.
//
// Warps: 0-7 softmax / epilogue (two warpgroups; thread (g, h) owns key
// columns 32g..32g+31 of every tile for head h, and latent columns
// 128g..128g+127 of O in the epilogue), 8 TMA producer, 9 MMA issuer and TMEM
// owner.  The two halves of a row agree on its max through shared memory
// once per tile.  The softmax runs one tile ahead on the
// exchange: it reads and sends the partial scores of tile j+1 before it
// finishes tile j, so the partner's data for a tile is usually there when it
// is needed.  It is online with a lazily updated reference max: O is rescaled
// only when a row max grows by more than 2^8.  Every wait is bounded; a wait
// that runs out raises the device error word and the CTA takes its exit path.
#pragma once

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kAttnThreads = 320;
constexpr int kSoftmaxThreads = 256;   // warps 0-7
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kTileN = 64;     // keys per tile
constexpr int kStages = 4;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct AttnLayout {
  static constexpr int kKvBox = kTileN * 128;           // 64 keys x 64 bf16 latent columns
  static constexpr int kKv = 4 * kKvBox;                // this CTA's 256 latent columns
  static constexpr int kPe = kTileN * 64;               // 64 keys x 32 bf16 rotary columns
  static constexpr int kStage = kKv + kPe;              // 36 KB, a multiple of 1024
  static constexpr int kQpe = 128 * 64;                 // 128 heads x 32 bf16
  static constexpr int kP = 128 * kTileN * 2;           // 128 heads x 64 keys bf16 = 16 KB
  static constexpr int kXchgSlot = 128 * kTileN * 2;    // 128 heads x 64 fp16 partial scores = 16 KB
  // P buffer, outbox and the two inbox slots are contiguous (64 KB).  Before
  // the first tile they are the landing zone of this CTA's q_abs half (4 boxes
  // of 128 heads x 64 latent columns, 16 KB each) on its way into TMEM.
  static constexpr int kOffQpe = kStages * kStage;
  static constexpr int kOffP = kOffQpe + kQpe;
  static constexpr int kOffOutbox = kOffP + kP;
  static constexpr int kOffInbox = kOffOutbox + kXchgSlot;
  static constexpr int kOffBars = kOffInbox + 2 * kXchgSlot;
  static constexpr int kOffMisc = kOffBars + 256;      // per-row max of each half [2 slots][2][128], sums [2][128]
  static constexpr int kBytes = kOffMisc + 4096;
  static constexpr int kAlloc = kBytes + 1024;          // room to align the base to 1024
};

struct AttnParams {
  const __nv_bfloat16* q_abs;   // [n_q, H, 512]
  const int* cu_q;              // [batch+1] for chunked prefill, nullptr for decode
  const int* cu_k;              // [batch+1]
  int batch;
  int heads;
  int head_groups;              // heads / 128
  int num_splits;
  int64_t kv_rows;
  int64_t n_q;
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* o_lat;         // [n_q, H, 512], written when num_splits == 1
  float* part_o;                // [splits, n_q, H, 512]
  float* part_ml;               // [splits, n_q, H, 2] = (reference max in log2 units, sum)
};

__device__ __forceinline__ uint32_t cvt_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 f16x2_to_f2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    latent_attn_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_pe,
                       const __grid_constant__ CUtensorMap tmap_qpe, const __grid_constant__ CUtensorMap tmap_qabs,
                       const AttnParams p) {
  using L = AttnLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qpe_s = smem + L::kOffQpe;
  uint8_t* p_s = smem + L::kOffP;
  uint8_t* xchg = smem + L::kOffP;      // q_abs landing zone = P + outbox + inbox
  uint8_t* outbox = smem + L::kOffOutbox;
  uint8_t* inbox = smem + L::kOffInbox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  // barrier slots, laid out from kStages so the ring depth can change safely
  uint64_t* kv_full = bars;                      // [kStages] TMA tile landed
  uint64_t* kv_empty = kv_full + kStages;        // [kStages] tile no longer read by the tensor core
  uint64_t* s_full = kv_empty + kStages;         // [2]  QK product committed
  uint64_t* s_free = s_full + 2;                 // [2]  softmax read S (256 arrivals)
  uint64_t* p_ready = s_free + 2;                // [2]  P written (256 arrivals)
  uint64_t* xchg_full = p_ready + 2;             // [2]  partner's partial scores landed in my inbox
  uint64_t* xchg_free = xchg_full + 2;           // [2]  partner's inbox slot is free (8 arrivals from its warps)
  uint64_t* outbox_ready = xchg_free + 2;        // [2]  all rows of my partial written (256 arrivals)
  uint64_t* mx_bar = outbox_ready + 2;           // [2]  both halves published their tile max (256 arrivals)
  uint64_t* o_done = mx_bar + 2;                 // one phase per P V product
  uint64_t* o_final = o_done + 1;                // the last P V product finished
  uint64_t* q_ready = o_final + 1;               // q_abs half stored in TMEM (256 arrivals)
  uint64_t* q_full = q_ready + 1;                // q_abs half landed in the exchange area
  uint64_t* qpe_full = q_full + 1;
  uint64_t* mma_idle = qpe_full + 1;             // every MMA of this CTA finished
  uint64_t* outbox_free = mma_idle + 1;          // the partner received my last copy (its MMA warp arrives)
  uint64_t* l_bar = outbox_free + 1;             // both halves published their sums (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(l_bar + 1);
  static_assert(2 * kStages + 22 + 1 <= 256 / 8, "barrier area too small");   // 8-byte slots incl. the TMEM address
  float* half_max = reinterpret_cast<float*>(smem + L::kOffMisc);          // [2][2][128]
  float* half_sum = half_max + 512;                                        // [2][128]

  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();
  const uint32_t rank = ptx::cluster_rank(), peer = rank ^ 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 1);
      ptx::mbar_init(&s_free[s], kSoftmaxThreads);
      ptx::mbar_init(&p_ready[s], kSoftmaxThreads);
      ptx::mbar_init(&xchg_full[s], 1);
      ptx::mbar_init(&xchg_free[s], kSoftmaxThreads / 32);
      ptx::mbar_init(&outbox_ready[s], kSoftmaxThreads);
      ptx::mbar_init(&mx_bar[s], kSoftmaxThreads);
    }
    ptx::mbar_init(l_bar, kSoftmaxThreads);
    ptx::mbar_init(outbox_free, 1);
    ptx::mbar_init(o_done, 1);
    ptx::mbar_init(o_final, 1);
    ptx::mbar_init(q_ready, kSoftmaxThreads);
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(qpe_full, 1);
    ptx::mbar_init(mma_idle, 1);
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  ptx::cluster_sync();   // the partner's barriers exist before anything remote touches them
  const uint32_t tmem = *tmem_slot;
  // set-up above touches no global memory; inputs may come from the previous kernel
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  // ---- work unit: (query row, head group, split) -------------------------
  const int64_t unit = blockIdx.x >> 1;
  const int per_row = p.head_groups * p.num_splits;
  const int64_t row = unit / per_row;
  const int hg = (int)((unit % per_row) / p.num_splits);
  const int sp = (int)(unit % p.num_splits);
  const int b = p.cu_q ? find_sequence(p.cu_q, p.batch, row) : (int)row;
  const int64_t k0 = min64(max64(0, __ldg(p.cu_k + b)), p.kv_rows);
  const int64_t t = max64(0, min64((int64_t)__ldg(p.cu_k + b + 1), p.kv_rows) - k0);
  int64_t visible = t;
  if (p.cu_q) {
    const int64_t q0 = __ldg(p.cu_q + b);
    const int64_t s = max64(0, (int64_t)__ldg(p.cu_q + b + 1) - q0);
    visible = min64(t, max64(0, t - s + (row - q0) + 1));
  }
  const int64_t per = ((visible + p.num_splits - 1) / p.num_splits + kTileN - 1) / kTileN * kTileN;
  const int64_t j_begin = min64(visible, (int64_t)sp * per);
  const int64_t j_end = min64(visible, j_begin + per);
  const int nt = (int)((j_end - j_begin + kTileN - 1) / kTileN);
  const int head0 = hg * 128;


  constexpr uint32_t kColO = 0, kColQ = 256, kColS = 384;

  if (warp == kProducerWarp) {
    // ================================================= TMA producer ======
    // The whole warp runs the loop (waits are warp-wide); one elected lane issues.
    int issued = 0;
    if (ptx::elect_one()) {
      ptx::prefetch_tmap(&tmap_kv);
      ptx::prefetch_tmap(&tmap_pe);
      if (nt > 0) {
        ptx::mbar_arrive_expect_tx(q_full, 4 * L::kXchgSlot);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          ptx::tma_load_2d(xchg + bx * L::kXchgSlot, &tmap_qabs, q_full, 256 * (int)rank + 64 * bx,
                           (int)(row * p.heads + head0));
        ptx::mbar_arrive_expect_tx(qpe_full, L::kQpe);
        ptx::tma_load_3d(qpe_s, &tmap_qpe, qpe_full, 128 + 32 * (int)rank, head0, (int)row);
      }
    }
    __syncwarp();
    for (int j = 0; j < nt; ++j) {
      const int s = j % kStages;
      const bool w = ptx::mbar_wait(&kv_empty[s], ((j / kStages) & 1) ^ 1, kErrTimeoutStageFree);
      if (!__all_sync(0xffffffffu, w)) break;
      if (ptx::elect_one()) {
        uint8_t* st = smem + s * L::kStage;
        ptx::mbar_arrive_expect_tx(&kv_full[s], L::kStage);
        const int key = (int)(k0 + j_begin + (int64_t)j * kTileN);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          ptx::tma_load_2d(st + bx * L::kKvBox, &tmap_kv, &kv_full[s], 256 * (int)rank + 64 * bx, key);
        ptx::tma_load_2d(st + L::kKv, &tmap_pe, &kv_full[s], 32 * (int)rank, key);
      }
      __syncwarp();
      issued = j + 1;
    }
    // exit path: every copy this CTA started has landed before its smem goes away
    for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
      ptx::mbar_wait(&kv_full[j % kStages], (j / kStages) & 1, kErrTimeoutDrain);
    if (nt > 0) {
      ptx::mbar_wait(qpe_full, 0, kErrTimeoutDrain);
      ptx::mbar_wait(q_full, 0, kErrTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================================================= MMA issuer ========
    // Two streams issued as their inputs arrive: QK(j) needs tile j and S
    // buffer j&1 read out (tile j-2); PV(j) needs P(j).  QK runs ahead of PV,
    // so the scores of the next tiles are ready while the softmax works.
    // The whole warp runs the loop with warp-uniform decisions; one elected
    // lane issues each MMA and commit.
    if (nt > 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(128, kTileN, false, false);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 256, false, true);
      bool ok = ptx::mbar_wait(q_ready, 0, kErrTimeoutSoftmax) && ptx::mbar_wait(qpe_full, 0, kErrTimeoutTmaFull);
      ok = __all_sync(0xffffffffu, ok);
      // descriptor bases; the start address sits in the low bits, so offsets add directly (>> 4)
      const uint64_t d_stage0 = ptx::smem_desc(ptx::smem_u32(smem), 16, 1024, ptx::kSwizzle128);
      const uint64_t d_pe0 = ptx::smem_desc(ptx::smem_u32(smem + L::kKv), 16, 512, ptx::kSwizzle64);
      const uint64_t d_qpe = ptx::smem_desc(ptx::smem_u32(qpe_s), 16, 512, ptx::kSwizzle64);
      const uint64_t d_p0 = ptx::smem_desc(ptx::smem_u32(p_s), 16, 1024, ptx::kSwizzle128);
      const uint64_t d_v0 = ptx::smem_desc(ptx::smem_u32(smem), L::kKvBox, 1024, ptx::kSwizzle128);
      int qk = 0, pv = 0, fw = 0;
      uint64_t t_last = global_timer_ns();
      ptx::tc_fence_after();
      // Third stream: as soon as the partner's copy of tile fw has landed in my
      // inbox, tell it (its single outbox may be refilled).  This must not wait
      // for the softmax: the softmax sends tile j+1 before it finishes tile j.
      while (ok && (pv < nt || fw < nt - 1)) {
        bool progressed = false;
        bool go_fw = fw < nt - 1 && ptx::mbar_test(&xchg_full[fw & 1], (fw >> 1) & 1);
        if (__shfl_sync(0xffffffffu, go_fw, 0)) {
          if (lane == 0) ptx::mbar_arrive_cluster_relaxed(outbox_free, peer);
          __syncwarp();
          ++fw;
          progressed = true;
        }
        bool go = qk < nt && (qk < 2 || ptx::mbar_test(&s_free[qk & 1], ((qk - 2) >> 1) & 1)) &&
                  ptx::mbar_test(&kv_full[qk % kStages], (qk / kStages) & 1);
        if (__shfl_sync(0xffffffffu, go, 0)) {
          ptx::tc_fence_after();
          const uint32_t so = (uint32_t)((qk % kStages) * L::kStage) >> 4;
          const uint32_t scol = tmem + kColS + (qk & 1) * kTileN;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            if (ptx::elect_one())
              ptx::mma_ts(scol, tmem + kColQ + ks * 8,
                          d_stage0 + so + (((ks >> 2) * L::kKvBox + (ks & 3) * 32) >> 4), idesc_qk,
                          ks > 0 ? 1u : 0u);
            __syncwarp();
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            if (ptx::elect_one()) ptx::mma_ss(scol, d_qpe + ((ks * 32) >> 4), d_pe0 + so + ((ks * 32) >> 4), idesc_qk, 1u);
            __syncwarp();
          }
          if (ptx::elect_one()) ptx::mma_commit(&s_full[qk & 1]);
          __syncwarp();
          ++qk;
          progressed = true;
        }
        go = pv < qk && ptx::mbar_test(&p_ready[pv & 1], (pv >> 1) & 1);
        if (__shfl_sync(0xffffffffu, go, 0)) {
          ptx::tc_fence_after();
          const uint32_t so = (uint32_t)((pv % kStages) * L::kStage) >> 4;
#pragma unroll
          for (int ks = 0; ks < kTileN / 16; ++ks) {
            if (ptx::elect_one())
              ptx::mma_ss(tmem + kColO, d_p0 + ((ks * 32) >> 4), d_v0 + so + ((ks * 2048) >> 4), idesc_pv,
                          (pv > 0 || ks > 0) ? 1u : 0u);
            __syncwarp();
          }
          if (ptx::elect_one()) {
            ptx::mma_commit(&kv_empty[pv % kStages]);
            ptx::mma_commit(o_done);
            if (pv == nt - 1) ptx::mma_commit(o_final);
          }
          __syncwarp();
          ++pv;
          progressed = true;
        }
        if (progressed) {
          t_last = global_timer_ns();
        } else {
          __nanosleep(20);
          bool late = global_timer_ns() - t_last > kWaitLimitNs;
          if (__shfl_sync(0xffffffffu, late, 0)) {
            if (lane == 0) raise_error(qk < nt ? kErrTimeoutTmaFull : kErrTimeoutSoftmax);
            ok = false;
          }
        }
      }
      // nothing of ours may still be running in the tensor core when TMEM is freed
      if (ptx::elect_one()) ptx::mma_commit(mma_idle);
      __syncwarp();
      ptx::mbar_wait(mma_idle, 0, kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ================================================= softmax (warps 0-7)
    const int g = (int)(warp >> 2);                    // half: key columns 32g.. of a tile, O columns 128g..
    const int h = (int)((warp & 3) * 32 + lane);       // head within the group = TMEM lane
    const uint32_t lane_base = (warp & 3) * 32u << 16;
    const int64_t head = head0 + h;
    const uint32_t sw = (uint32_t)(h & 7);             // 128-byte swizzle phase of row h
    bool ok = true;
    float m_ref = -INFINITY, l = 0.f;                  // l: this half's share of the row sum
    if (nt > 0) {
      // this CTA's half of q_abs: exchange area (TMA, 128-byte swizzle) -> TMEM columns [256, 384)
      bool w = ptx::mbar_wait(q_full, 0, kErrTimeoutTmaFull);
      ok = __all_sync(0xffffffffu, w);
      if (ok) {
#pragma unroll 1
        for (int c = 2 * g; c < 2 * g + 2; ++c) {
          const uint8_t* src = xchg + c * L::kXchgSlot + h * 128;
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = *reinterpret_cast<const uint4*>(src + ((v ^ sw) << 4));
            r[4 * v] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
          }
          ptx::tmem_st32(tmem + lane_base + kColQ + c * 32, r);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(q_ready);
        // every softmax thread has read its part of the landing zone before any is reused
        w = ptx::mbar_wait(q_ready, 0, kErrTimeoutSoftmax);
        ok = __all_sync(0xffffffffu, w);
      }
      if (ok) {
        // the inbox is free again: the partner may send into it
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive_cluster_relaxed(&xchg_free[0], peer);
          ptx::mbar_arrive_cluster_relaxed(&xchg_free[1], peer);
        }
      }

      const uint32_t peer_inbox = ptx::map_peer(ptx::smem_u32(inbox), peer);
      const uint32_t peer_full0 = ptx::map_peer(ptx::smem_u32(&xchg_full[0]), peer);
      const uint32_t peer_full1 = ptx::map_peer(ptx::smem_u32(&xchg_full[1]), peer);
      const float sl2 = p.scale_log2;

      // Send: my 32 partial scores of tile j (TMEM -> fp16 -> outbox -> one bulk
      // copy of the whole outbox into the partner's inbox); kept in `own`.
      auto send = [&](int j, uint32_t (&own)[16]) -> bool {
        const int slot = j & 1;
        const uint32_t par = (j >> 1) & 1;
        bool w = ptx::mbar_wait(&s_full[slot], par, kErrTimeoutMma);
        if (!__all_sync(0xffffffffu, w)) return false;
        ptx::tc_fence_after();
        {
          uint32_t a[32];
          ptx::tmem_ld32(tmem + lane_base + kColS + slot * kTileN + 32 * g, a);
          ptx::tmem_wait_ld();
          ptx::tc_fence_before();
          ptx::mbar_arrive(&s_free[slot]);               // S buffer may take QK(j+2)
#pragma unroll
          for (int i = 0; i < 16; ++i) own[i] = cvt_f16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
        }
        w = ptx::mbar_wait<true>(&xchg_free[slot], par, kErrTimeoutPeer);
        // the outbox is free once the partner has received my previous copy
        if (j >= 1) w = w && ptx::mbar_wait<true>(outbox_free, (j - 1) & 1, kErrTimeoutPeer);
        if (!__all_sync(0xffffffffu, w)) return false;
        uint8_t* dst = outbox + h * 128;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(dst + (((4 * g + k) ^ sw) << 4)) =
              make_uint4(own[4 * k], own[4 * k + 1], own[4 * k + 2], own[4 * k + 3]);
        ptx::fence_async_smem();
        ptx::mbar_arrive(&outbox_ready[slot]);
        if (threadIdx.x == 0) {
          // every row is in the outbox (a bounded wait, unlike a named barrier) -> one bulk copy
          if (ptx::mbar_wait(&outbox_ready[slot], par, kErrTimeoutSoftmax))
            ptx::bulk_copy_to_peer(peer_inbox + slot * L::kXchgSlot, ptx::smem_u32(outbox), L::kXchgSlot,
                                   slot ? peer_full1 : peer_full0);
          ptx::mbar_arrive_expect_tx(&xchg_full[slot], L::kXchgSlot);
        }
        return true;
      };

      // Finish tile j: add the partner's partial, online softmax, P into shared memory.
      auto finish = [&](int j, const uint32_t (&own)[16]) -> bool {
        const int slot = j & 1;
        const uint32_t par = (j >> 1) & 1;
        bool w = ptx::mbar_wait<true>(&xchg_full[slot], par, kErrTimeoutPeer);
        if (!__all_sync(0xffffffffu, w)) return false;
        // raw scores: my fp16 partial + the partner's fp16 partial (packed fp16 adds)
        uint32_t sum2[16];
        {
          const uint8_t* mine = inbox + slot * L::kXchgSlot + h * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 v = *reinterpret_cast<const uint4*>(mine + (((4 * g + k) ^ sw) << 4));
            const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __half2 a = *reinterpret_cast<const __half2*>(&own[4 * k + e]);
              __half2 c = *reinterpret_cast<const __half2*>(&pv[e]);
              __half2 r = __hadd2(a, c);
              sum2[4 * k + e] = *reinterpret_cast<uint32_t*>(&r);
            }
          }
        }
        const int64_t key0 = j_begin + (int64_t)j * kTileN;
        const int n_valid = (int)min64(kTileN, j_end - key0);
        const int c0 = 32 * g;                           // first key column of this half
        if (n_valid < kTileN) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // keys past the end: -inf (fp16 0xFC00) in the masked half(s)
            if (c0 + 2 * i >= n_valid) sum2[i] = 0xFC00FC00u;
            else if (c0 + 2 * i + 1 >= n_valid) sum2[i] = (sum2[i] & 0x0000FFFFu) | 0xFC000000u;
          }
        }
        float hm;
        {
          __half2 m4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __half2* v = reinterpret_cast<const __half2*>(&sum2[4 * i]);
            m4[i] = __hmax2(__hmax2(v[0], v[1]), __hmax2(v[2], v[3]));
          }
          const __half2 m2 = __hmax2(__hmax2(m4[0], m4[1]), __hmax2(m4[2], m4[3]));
          hm = fmaxf(__low2float(m2), __high2float(m2)) * sl2;   // scale >= 0
        }
        // the row max is the max of the two halves' maxima
        half_max[(slot * 2 + g) * 128 + h] = hm;
        ptx::mbar_arrive(&mx_bar[slot]);
        w = ptx::mbar_wait(&mx_bar[slot], par, kErrTimeoutSoftmax);
        if (!__all_sync(0xffffffffu, w)) return false;
        const float mx = fmaxf(hm, half_max[(slot * 2 + (g ^ 1)) * 128 + h]);
        // the P buffer and O are only touched once the P V product of tile j-1 is done
        if (j >= 1) {
          w = ptx::mbar_wait(o_done, (j - 1) & 1, kErrTimeoutMma);
          if (!__all_sync(0xffffffffu, w)) return false;
          ptx::tc_fence_after();
        }
        if (j == 0) {
          m_ref = mx;
        } else {
          const bool grow = mx > m_ref + kRescaleThreshold;
          // Both halves of a row see the same mx, so they agree on the rescale.
          // TMEM loads/stores are warp-wide: the warp rescales together, lanes
          // whose row max did not grow use factor 1.  Half g rescales O[:, 128g..].
          if (__any_sync(0xffffffffu, grow)) {
            const float f = grow ? fast_exp2(m_ref - mx) : 1.f;
            l *= f;
#pragma unroll 1
            for (int c = 4 * g; c < 4 * g + 4; ++c) {
              uint32_t r[32];
              ptx::tmem_ld32(tmem + lane_base + kColO + c * 32, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
              ptx::tmem_st32(tmem + lane_base + kColO + c * 32, r);
            }
            ptx::tmem_wait_st();
            if (grow) m_ref = mx;
          }
        }
        // P = 2^(s*scale*log2e - m_ref) as bf16, keys 32g.. of row h of the K-major P tile (128-byte swizzle)
        uint8_t* prow = p_s + h * 128;
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t q4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xs = __half22float2(*reinterpret_cast<const __half2*>(&sum2[4 * k + e]));
            float e0 = fast_exp2(fmaf(xs.x, sl2, -m_ref));
            float e1 = fast_exp2(fmaf(xs.y, sl2, -m_ref));
            if (n_valid < kTileN) {   // keys past the end weigh exactly 0 (also when scale is 0)
              if (c0 + 8 * k + 2 * e >= n_valid) e0 = 0.f;
              if (c0 + 8 * k + 2 * e + 1 >= n_valid) e1 = 0.f;
            }
            ps[e] += e0 + e1;
            q4[e] = ptx::pack_bf16x2(e0, e1);
          }
          *reinterpret_cast<uint4*>(prow + (((4 * g + k) ^ sw) << 4)) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
        }
        l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        if (n_valid < kTileN) {
          // keys past the end get P = 0, but 0 * NaN is NaN: clear their latent rows
          uint8_t* st = smem + (j % kStages) * L::kStage;
          const int rows = kTileN - n_valid;
          for (int idx = (int)threadIdx.x; idx < rows * 4 * 8; idx += kSoftmaxThreads) {
            const int bx = idx / (rows * 8), rem = idx % (rows * 8);
            *reinterpret_cast<uint4*>(st + bx * L::kKvBox + (n_valid + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        ptx::fence_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_ready[slot]);
        // my inbox slot is consumed: the partner may send tile j+2 into it
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster_relaxed(&xchg_free[slot], peer);
        return true;
      };

      uint32_t cur[16], nxt[16];
      if (ok) ok = send(0, cur);
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          ok = send(j + 1, nxt);
          if (!ok) break;
        }
        ok = finish(j, cur);
#pragma unroll
        for (int i = 0; i < 16; ++i) cur[i] = nxt[i];
      }
    }

    // ---- epilogue ----------------------------------------------------------
    // thread (g, h) writes latent columns 256*rank + 128g .. +127 of head h
    const int64_t out_row = (row * p.heads + head) * 512 + 256 * rank + 128 * g;
    if (nt == 0) {
      if (p.num_splits == 1) {
        uint4* dst = reinterpret_cast<uint4*>(p.o_lat + out_row);
        for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      } else if (rank == 0 && g == 0) {
        float* ml = p.part_ml + (((int64_t)sp * p.n_q + row) * p.heads + head) * 2;
        ml[0] = -INFINITY;
        ml[1] = 0.f;
      }
    } else if (ok) {
      // the row sum is the sum of the two halves' sums
      half_sum[g * 128 + h] = l;
      ptx::mbar_arrive(l_bar);
      bool w = ptx::mbar_wait(l_bar, 0, kErrTimeoutSoftmax) && ptx::mbar_wait(o_final, 0, kErrTimeoutMma);
      if (__all_sync(0xffffffffu, w)) {
        const float lsum = half_sum[h] + half_sum[128 + h];
        ptx::tc_fence_after();
        if (p.num_splits == 1) {
          const float inv = 1.f / lsum;
          uint4* dst = reinterpret_cast<uint4*>(p.o_lat + out_row);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base + kColO + (4 * g + c) * 32, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t q4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                q4[e] = ptx::pack_bf16x2(__uint_as_float(r[8 * v + 2 * e]) * inv,
                                         __uint_as_float(r[8 * v + 2 * e + 1]) * inv);
              dst[c * 4 + v] = make_uint4(q4[0], q4[1], q4[2], q4[3]);
            }
          }
        } else {
          const int64_t slot = ((int64_t)sp * p.n_q + row) * p.heads + head;
          float4* dst = reinterpret_cast<float4*>(p.part_o + slot * 512 + 256 * rank + 128 * g);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base + kColO + (4 * g + c) * 32, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[c * 8 + v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                           __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          }
          if (rank == 0 && g == 0) {
            p.part_ml[slot * 2] = m_ref;
            p.part_ml[slot * 2 + 1] = lsum;
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, 512);
  ptx::cluster_sync();   // the partner no longer writes into this CTA's shared memory
}

// Merge split partials: o = sum_s 2^{m_s - M} o_s / sum_s 2^{m_s - M} l_s, M = max_s m_s.
// One block of 128 threads per (row, head); warp 0 turns the (m, l) pairs into
// weights, then thread i accumulates columns 4i..4i+3 over the splits with
// several loads in flight.  Splits with no key (m = -inf) get weight 0 and
// their (unwritten) partial is never used.
constexpr int kMaxSplits = 256;
__global__ void __launch_bounds__(128) merge_splits_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_ml, int num_splits,
                                                           int64_t n_q, int heads, __nv_bfloat16* __restrict__ o_lat) {
  __shared__ float s_w[kMaxSplits];
  __shared__ float s_inv;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t row = blockIdx.x;
  const int head = blockIdx.y;
  const int64_t split_stride = n_q * heads;
  const int64_t base = row * heads + head;
  if (threadIdx.x < 32) {
    float M = -INFINITY;
    for (int s = threadIdx.x; s < num_splits; s += 32) M = fmaxf(M, part_ml[(s * split_stride + base) * 2]);
    M = warp_max(M);
    float L = 0.f;
    for (int s = threadIdx.x; s < num_splits; s += 32) {
      const float ms = part_ml[(s * split_stride + base) * 2];
      const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
      s_w[s] = w;
      L += w * part_ml[(s * split_stride + base) * 2 + 1];
    }
    L = warp_sum(L);
    if (threadIdx.x == 0) s_inv = L > 0.f ? 1.f / L : 0.f;
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* src = reinterpret_cast<const float4*>(part_o + base * 512) + threadIdx.x;
  const int64_t step = split_stride * 512 / 4;
#pragma unroll 8
  for (int s = 0; s < num_splits; ++s) {
    const float w = s_w[s];
    const float4 v = src[s * step];
    if (w != 0.f) {
      acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
    }
  }
  const float inv = s_inv;
  uint2 o;
  o.x = ptx::pack_bf16x2(acc.x * inv, acc.y * inv);
  o.y = ptx::pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(o_lat + base * 512)[threadIdx.x] = o;
}

}  // namespace sm100
}  // namespace mla
