// sm100_attn.cuh -- latent attention on tcgen05 for the DeepSeek-V3 shapes
// (C = 512 latent columns, R = 64 rotary columns, 128 heads per row block).
//
// Operation ("Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Absorb Path Execution"): for one query row and 128 heads
//   S[h,t] = (q_abs[h,:] . kv[t,:] + q_pe[h,:] . pe[t,:]) * scale
//   P      = softmax_t(S)   (keys past the row's visible limit masked)
//   o[h,:] = sum_t P[h,t] kv[t,:]
// The latent cache is both key and value.
//
// Why two CTAs: the fp32 accumulator O for 128 heads x 512 columns is 256 KB,
// all of one SM's tensor memory, and the query needs 256 more columns.  So a
// work unit runs on a cluster of two CTAs with fixed roles and a one-way
// hand-off:
//
//   score CTA (rank 0): q_abs in TMEM, S = Q K^T over all 576 contraction
//     columns for 128 keys at a time (36 tcgen05.mma with N = 128), the
//     online softmax, and P (bf16, 64 keys at a time) staged in shared memory and
//     sent to the value CTA with one bulk copy per warp.
//   value CTA (rank 1): O in TMEM, O += P V (8 tcgen05.mma with N = 256 per
//     64 keys, A = P and B = the kv tile, both from shared memory), the rare O
//     rescale, and the epilogue (O or the split partial as bf16).
//
// The score CTA never waits for the value CTA except for a free P slot (four
// slots), so the pair forms a pipeline instead of exchanging partial scores
// every tile.  Each CTA streams its own copy of the kv rows: the score CTA
// from HBM, the value CTA a little later from L2, so HBM sees each cache byte
// once.  N = 128 matters: with one
// elected lane issuing, a 128 x 64 x 16 MMA takes 48 cycles where 32 would be
// full rate, while N >= 128 runs at full rate.
//
// Score CTA.  TMEM: [0,256) q_abs (bf16 pairs; it lands by TMA in latent
// slots 1-4 and the softmax threads move it into TMEM), two S buffers of 128
// columns at 256 and 384.  Shared memory (128-byte swizzle throughout): a ring
// of five 32 KB latent slots (two 64-column blocks of 128 keys, one TMA copy
// each; four make the latent part of a score tile), two 16 KB rotary slots
// (the 64 rotary columns of 128 keys), q_pe (128 heads x 64, the A operand of
// the rotary products) and one P staging slot.  A copy costs the TMA engine a
// fixed overhead besides its bytes, so fewer, larger copies per tile raise the
// rate at which one SM can pull keys.  Warps 0-3 and 4-7 are two softmax warpgroups that take
// alternate score tiles (thread = head row, all 128 keys); warp 8 loads,
// warp 9 issues the MMAs.  The running reference max m of each row passes
// from one warpgroup to the other once per tile through shared memory; it is
// updated lazily (only when a tile's max exceeds it by more than 2^8), so
// P <= 256.  When it moves, the factor 2^(m_old - m_new) travels with P and
// the value CTA rescales O before the next P V product.
//
// Value CTA.  TMEM: O, all 512 columns.  Shared memory: a 2-stage ring of
// 64-key kv tiles (eight 8 KB boxes; they hit L2, the score CTA read the rows
// first) and four P slots (P 16 KB, the per-row factor, and in slot 0 the
// final row sums).  Warps 0-3 check each tile's
// factors (and rescale O when one moved), zero the tail rows of the last
// tile's values, and release the P V product; warp 8 loads, warp 9 issues
// the MMAs and hands P slots back; warps 0-7 run the epilogue.
//
// The cache is packed (sequence b's keys in rows cu_k[b] ..) or paged: key j
// of sequence b in row table[b][j / page] * page + j % page, pages of a
// multiple of 64 keys ("What is DeepSeek Sparse Attention (DSA)?", section
// "How DSA works (conceptual)": the serving runtime keeps the KV cache in
// pages for continuous batching).  Paging changes only which rows the copies
// start at (CacheRows); with pages of 64 * odd keys a 128-key score copy
// becomes two 64-key copies.
//
// Every wait is bounded; a wait that runs out raises the device error word
// and the thread takes its exit path.
#pragma once

#include "sm100_ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kAttnThreads = 320;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kTileN = 64;                 // keys per P tile (value CTA granule)
constexpr int kTileQ = 128;                // keys per score tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Score CTA shared memory.
struct ScoreLayout {
  static constexpr int kBlock = kTileQ * 128;              // 128 keys x 64 columns bf16 (16 KB)
  static constexpr int kLat = 2 * kBlock;                  // latent slot: two 64-column blocks (one TMA copy)
  static constexpr int kLatSlots = 5;
  static constexpr int kLatPerTile = 4;
  static constexpr int kPeSlots = 2;
  static constexpr int kOffPe = kLatSlots * kLat;          // rotary slots, 16 KB each
  static constexpr int kOffQpe = kOffPe + kPeSlots * kBlock;  // q_pe: 128 heads x 64 bf16
  static constexpr int kOffStaging = kOffQpe + 128 * 128;  // the P staging slot, laid out like the value CTA's
  static constexpr int kSlot = 17408;                      // P 16 KB, factors 512 B
  static constexpr int kOffM = kOffStaging + kSlot;        // reference max published by warpgroup g: [2][128]
  static constexpr int kOffEndL = kOffM + 1024;            // warpgroup 1's row sums at the end [128]
  static constexpr int kOffBars = kOffEndL + 512;
  static constexpr int kBytes = kOffBars + 512;
  static constexpr int kOffQ = kLat;                       // q_abs lands in latent slots 1-4 (128 KB)
};

// Value CTA shared memory.
struct ValueLayout {
  static constexpr int kKvBox = kTileN * 128;              // 64 keys x 64 latent columns bf16
  static constexpr int kStage = 8 * kKvBox;                // 64 keys x 512 latent columns
  static constexpr int kStages = 2;
  static constexpr int kPSlots = 4;
  static constexpr int kOffSlots = kStages * kStage;       // P slots
  static constexpr int kSlot = 17408;                      // 1024-aligned
  static constexpr int kP = 128 * kTileN * 2;              // P: 128 heads x 64 keys bf16, 16 KB
  static constexpr int kOffF = kP;                         // in a slot: the per-row factors, 512 B
  static constexpr int kOffL = kOffSlots + kP + 512;       // in slot 0: the final row sums, 512 B
  static constexpr int kOffBars = kOffSlots + kPSlots * kSlot;
  static constexpr int kBytes = kOffBars + 512;
};

constexpr int kAttnSmem = ScoreLayout::kBytes > ValueLayout::kBytes ? ScoreLayout::kBytes : ValueLayout::kBytes;
static_assert(kAttnSmem <= 232448, "attention shared memory above the per-CTA limit");
static_assert(ScoreLayout::kOffPe % 1024 == 0 && ScoreLayout::kOffQpe % 1024 == 0 && ScoreLayout::kOffStaging % 1024 == 0 &&
                  ValueLayout::kOffSlots % 1024 == 0 && ValueLayout::kSlot % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
static_assert(ScoreLayout::kSlot == ValueLayout::kSlot, "staging and P slots share one layout");
static_assert(ValueLayout::kP + 1024 <= ValueLayout::kSlot, "P slot too small");

struct AttnParams {
  const __nv_bfloat16* q_abs;   // [n_q, H, 512]
  const int* cu_q;              // [batch+1] for chunked prefill, nullptr for decode
  const int* cu_k;              // [batch+1] packed cache: first row of each sequence
  const int* seqlens_k;         // [batch] paged cache: keys per sequence
  const int* block_table;       // [batch, bt_stride] paged cache: page of each run of page_size keys;
                                // nullptr for a packed cache
  int64_t bt_stride;
  int page_size;                // rows per page, a multiple of 64
  int score_copy_rows;          // keys per score-side copy: 128, or 64 when pages are 64 * odd
  int batch;
  int heads;
  int head_groups;              // heads / 128
  int num_splits;
  int partials;                 // 1: write the split partial form (O relative to m, and (m, l)) even for one split
  int early_cache;              // 1: the value CTA starts its cache stream before waiting for the previous kernel
  int64_t kv_rows;
  int64_t n_q;
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* o_lat;         // [n_q, H, 512]
  __nv_bfloat16* out;           // the epilogue's rows of 512: o_lat, or the split partials [splits * n_q * H, 512]
  float* part_ml;               // [splits, n_q, H, 2] = (reference max in log2 units, row sum)
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A unit's query row, head group, split and key range [j_begin, j_end) within
// its sequence (whose first cache row is k0); nt = number of 64-key P tiles.
struct UnitRange {
  int64_t row, k0, j_begin, j_end;
  int b, hg, sp, nt;
};

__device__ __forceinline__ UnitRange unit_range(const AttnParams& p, int64_t unit) {
  UnitRange u;
  const int per_row = p.head_groups * p.num_splits;
  u.row = unit / per_row;
  u.hg = (int)((unit % per_row) / p.num_splits);
  u.sp = (int)(unit % p.num_splits);
  const int b = p.cu_q ? find_sequence(p.cu_q, p.batch, u.row) : (int)u.row;
  u.b = b;
  int64_t t;
  if (p.block_table) {
    // keys are addressed through the block table (CacheRows); a sequence holds at most as
    // many keys as its row of the table has pages for
    u.k0 = 0;
    t = max64(0, min64((int64_t)__ldg(p.seqlens_k + b), p.bt_stride * p.page_size));
  } else {
    u.k0 = min64(max64(0, __ldg(p.cu_k + b)), p.kv_rows);
    t = max64(0, min64((int64_t)__ldg(p.cu_k + b + 1), p.kv_rows) - u.k0);
  }
  int64_t visible = t;
  if (p.cu_q) {
    // query i of s new queries (aligned to the end of the cache) sees keys 0 .. t - s + i
    const int64_t q0 = __ldg(p.cu_q + b);
    const int64_t s = max64(0, (int64_t)__ldg(p.cu_q + b + 1) - q0);
    visible = min64(t, max64(0, t - s + (u.row - q0) + 1));
  }
  // splits are whole score tiles
  const int64_t per = ((visible + p.num_splits - 1) / p.num_splits + kTileQ - 1) / kTileQ * kTileQ;
  u.j_begin = min64(visible, (int64_t)u.sp * per);
  u.j_end = min64(visible, u.j_begin + per);
  u.nt = (int)((u.j_end - u.j_begin + kTileN - 1) / kTileN);
  return u;
}

// Cache row of each key a unit loads, for one warp whose lanes all ask for the same key, keys
// non-decreasing from call to call.  Packed cache: the sequence's first row plus the key.
// Paged cache: key j of sequence b sits in row table[b][j / page] * page + j % page.  Lane l
// holds the table entry of page win + l, and the next 32 entries are already loading when the
// window moves on, so the copies wait on the table only once, at the start.  The packed
// form (kPaged = false) compiles to the first row plus the key and nothing else.
template <bool kPaged>
struct CacheRows {
  const int* bt;        // the sequence's row of the block table, nullptr for a packed cache
  int64_t base;         // packed cache: the sequence's first row
  int64_t n_entries;    // entries in the table row
  int64_t rows;         // cache rows
  int64_t win;
  int page, cur, nxt;

  __device__ __forceinline__ int entry(int64_t i) const { return i < n_entries ? __ldg(bt + i) : -1; }

  __device__ __forceinline__ void init(const AttnParams& p, const UnitRange& u, uint32_t lane) {
    base = u.k0;
    bt = nullptr;
    if (!kPaged) return;
    bt = p.block_table + (int64_t)u.b * p.bt_stride;
    rows = p.kv_rows;
    n_entries = p.bt_stride;
    page = p.page_size;
    win = u.j_begin / page;
    cur = entry(win + lane);
    nxt = entry(win + 32 + lane);
  }

  // Row of key j (counted from the sequence's first key).  A page outside the cache gives row
  // `rows`, past the end of the tensor maps, which the copies fill with zeros; when the page
  // holds a key the unit attends to (j < j_end) the device error word records it.
  __device__ __forceinline__ int row(int64_t j, int64_t j_end, uint32_t lane) {
    if (!kPaged) return (int)(base + j);
    const int64_t pg = j / page;
    while (pg >= win + 32) {
      cur = nxt;
      win += 32;
      nxt = entry(win + 32 + lane);
    }
    const int e = __shfl_sync(0xffffffffu, cur, (int)(pg - win));
    if (e < 0 || ((int64_t)e + 1) * page > rows) {
      if (j < j_end && lane == 0) raise_error(kErrBadPage);
      return (int)rows;
    }
    return (int)((int64_t)e * page + j % page);
  }
};

// Barrier slots (8 bytes each) in the 512-byte barrier area of either role.
namespace bar {
// score CTA
constexpr int kUFull = 0, kUEmpty = 5, kPeFull = 10, kPeEmpty = 12, kSFull = 22, kSFree = 24, kMBar = 26,
              kPFree = 28, kQFull = 32, kQReady = 33, kEnd = 34, kScoreIdle = 35, kPSent = 36, kQPiece = 14,
              kQFree = 18;
// value CTA
constexpr int kVFull = 0, kVEmpty = 2, kPFull = 4, kPvGo = 8, kPDone = 12, kOFinal = 16, kLFull = 17,
              kValueIdle = 18;
constexpr int kTmemSlot = 63;
}  // namespace bar

constexpr uint32_t kColQ = 0, kColS = 256;

// ---------------------------------------------------------------- score CTA
template <bool kPaged>
__device__ __forceinline__ void score_role(uint8_t* smem, uint32_t tmem, const UnitRange& u, const AttnParams& p,
                                           const CUtensorMap* tmap_kv, const CUtensorMap* tmap_pe,
                                           const CUtensorMap* tmap_qpe, const CUtensorMap* tmap_qabs) {
  using L = ScoreLayout;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  uint64_t* u_full = bars + bar::kUFull;       // [5] latent slot landed
  uint64_t* u_empty = bars + bar::kUEmpty;     // [5] latent slot read by the tensor core
  uint64_t* pe_full = bars + bar::kPeFull;     // [2] rotary slot landed
  uint64_t* pe_empty = bars + bar::kPeEmpty;   // [2] rotary slot read by the tensor core
  uint64_t* s_full = bars + bar::kSFull;       // [2] QK product committed
  uint64_t* s_free = bars + bar::kSFree;       // [2] S read out (128 arrivals)
  uint64_t* m_bar = bars + bar::kMBar;         // [2] warpgroup g published the reference max of its tile (128)
  uint64_t* p_free = bars + bar::kPFree;       // [4] the value CTA finished the P V product of this P slot
  uint64_t* q_full = bars + bar::kQFull;       // q_pe landed
  uint64_t* q_piece = bars + bar::kQPiece;     // [4] q_abs blocks 2k, 2k+1 landed in latent slot 1 + k
  uint64_t* q_free = bars + bar::kQFree;       // [4] those blocks moved into TMEM: slot 1 + k free (128 arrivals)
  uint64_t* q_ready = bars + bar::kQReady;     // all of q_abs in TMEM (256 arrivals)
  uint64_t* end_bar = bars + bar::kEnd;        // warpgroup 1 published its (l, m) (128)
  uint64_t* p_sent = bars + bar::kPSent;       // [2] warpgroup g stored the P tiles of its score tile (4 warps)
  uint64_t* idle = bars + bar::kScoreIdle;
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();
  const int ntp = u.nt;                        // 64-key P tiles
  const int ntq = (ntp + 1) / 2;               // 128-key score tiles
  const int head0 = u.hg * 128;

  if (warp == kProducerWarp) {
    // ============================================================ producer
    // q comes from the previous kernel
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    int lat_issued = 0, pe_issued = 0;
    if (ntp > 0) {
      if (ptx::elect_one()) {
        ptx::prefetch_tmap(tmap_kv);
        ptx::prefetch_tmap(tmap_pe);
        // q_pe, and q_abs (eight 64-column blocks of 128 heads) in four 32 KB pieces into latent
        // slots 1-4: each slot returns to the cache stream as soon as its piece is in TMEM
        ptx::mbar_arrive_expect_tx(q_full, 128 * 128);
        ptx::tma_load_3d(smem + L::kOffQpe, tmap_qpe, q_full, 128, head0, (int)u.row);
        for (int k = 0; k < 4; ++k) {
          ptx::mbar_arrive_expect_tx(&q_piece[k], L::kLat);
          ptx::tma_load_3d(smem + L::kOffQ + k * L::kLat, tmap_qabs, &q_piece[k], 0, (int)(u.row * p.heads + head0),
                           2 * k);
        }
      }
      __syncwarp();
      CacheRows<kPaged> cache;
      cache.init(p, u, lane);
      // pages of 64 * odd keys: each 128-key tile is two 64-key copies (rows r0, r1) per block
      const bool halves = kPaged && p.score_copy_rows != kTileQ;
      bool ok = true;
      for (int jj = 0; ok && jj < ntq; ++jj) {
        const int64_t j0 = u.j_begin + (int64_t)jj * kTileQ;
        const int r0 = cache.row(j0, u.j_end, lane);
        const int r1 = halves ? cache.row(j0 + kTileQ / 2, u.j_end, lane) : 0;
        // the rotary block of the tile
        const int ps = jj % L::kPeSlots;
        bool w = ptx::mbar_wait(&pe_empty[ps], ((jj / L::kPeSlots) & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) break;
        // (fault-injection builds only: a planned fault drops this copy, so the waits on it run out)
        const bool dropped = jj == 0 && u.row == 0 && u.hg == 0 && u.sp == 0 && fault_plan(1u);
        if (!dropped && ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(&pe_full[ps], L::kBlock);
          uint8_t* dst = smem + L::kOffPe + ps * L::kBlock;
          ptx::tma_load_2d(dst, tmap_pe, &pe_full[ps], 0, r0);
          if (halves) ptx::tma_load_2d(dst + L::kBlock / 2, tmap_pe, &pe_full[ps], 0, r1);
        }
        __syncwarp();
        pe_issued = jj + 1;
        // the latent blocks, two per copy
#pragma unroll 1
        for (int k = 0; k < L::kLatPerTile; ++k) {
          const int li = L::kLatPerTile * jj + k, slot = li % L::kLatSlots, use = li / L::kLatSlots;
          w = true;
          if (use == 0 && slot >= 1) w = ptx::mbar_wait(&q_free[slot - 1], 0, kErrTimeoutSoftmax);   // held q_abs
          w = w && ptx::mbar_wait(&u_empty[slot], (use & 1) ^ 1, kErrTimeoutStageFree);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          if (ptx::elect_one()) {
            ptx::mbar_arrive_expect_tx(&u_full[slot], L::kLat);
            uint8_t* dst = smem + slot * L::kLat;
            if (!halves) {
              ptx::tma_load_3d(dst, tmap_kv, &u_full[slot], 0, r0, 2 * k);
            } else {
              // 64 keys x 64 columns per copy; the 8 KB offsets keep the 128-byte swizzle phase
              for (int blk = 0; blk < 2; ++blk) {
                ptx::tma_load_3d(dst + blk * L::kBlock, tmap_kv, &u_full[slot], 0, r0, 2 * k + blk);
                ptx::tma_load_3d(dst + blk * L::kBlock + L::kBlock / 2, tmap_kv, &u_full[slot], 0, r1, 2 * k + blk);
              }
            }
          }
          __syncwarp();
          lat_issued = li + 1;
        }
      }
      // exit path: every copy this CTA started has landed before its shared memory goes away
      for (int li = (lat_issued > L::kLatSlots ? lat_issued - L::kLatSlots : 0); li < lat_issued; ++li)
        ptx::mbar_wait(&u_full[li % L::kLatSlots], (li / L::kLatSlots) & 1, kErrTimeoutDrain);
      for (int jj = (pe_issued > L::kPeSlots ? pe_issued - L::kPeSlots : 0); jj < pe_issued; ++jj)
        ptx::mbar_wait(&pe_full[jj % L::kPeSlots], (jj / L::kPeSlots) & 1, kErrTimeoutDrain);
      ptx::mbar_wait(q_full, 0, kErrTimeoutDrain);
      for (int k = 0; k < 4; ++k) ptx::mbar_wait(&q_piece[k], 0, kErrTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ============================================================ MMA issuer
    if (ntp > 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kTileQ, false, false);
      bool ok = ptx::mbar_wait(q_ready, 0, kErrTimeoutSoftmax) && ptx::mbar_wait(q_full, 0, kErrTimeoutTmaFull);
      ok = __all_sync(0xffffffffu, ok);
      // K-major operands, 128-byte rows, 8-row groups 1024 bytes apart; the start
      // address sits in the low bits, so byte offsets add directly (>> 4)
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(smem), 16, 1024, ptx::kSwizzle128);
      const uint64_t d_qpe = ptx::smem_desc(ptx::smem_u32(smem + L::kOffQpe), 16, 1024, ptx::kSwizzle128);
      ptx::tc_fence_after();
      // Each issue site has one fixed MMA form (the block loops are unrolled):
      // a loop that can reach both the TMEM-A and the shared-memory-A form from one
      // elected branch issued at a quarter of the tensor-core rate.
      for (int jj = 0; ok && jj < ntq; ++jj) {
        if (jj >= 2) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s_free[jj & 1], ((jj - 2) >> 1) & 1, kErrTimeoutSoftmax));
          if (!ok) break;
        }
        const uint32_t scol = tmem + kColS + (uint32_t)(jj & 1) * kTileQ;
        // rotary block first (it starts the accumulation): A = q_pe in shared memory
        {
          const int ps = jj % L::kPeSlots;
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(&pe_full[ps], (jj / L::kPeSlots) & 1, kErrTimeoutTmaFull));
          if (!ok) break;
          ptx::tc_fence_after();
          const uint64_t d_b = d_ring + (uint32_t)((L::kOffPe + ps * L::kBlock) >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (ptx::elect_one())
              ptx::mma_ss(scol, d_qpe + (uint32_t)((k * 32) >> 4), d_b + (uint32_t)((k * 32) >> 4), idesc,
                          k > 0 ? 1u : 0u);
            __syncwarp();
          }
          if (ptx::elect_one()) ptx::mma_commit(&pe_empty[ps]);
          __syncwarp();
        }
        // latent blocks: A = q_abs columns 64b.. in TMEM
#pragma unroll
        for (int k = 0; k < L::kLatPerTile; ++k) {
          const int li = L::kLatPerTile * jj + k, slot = li % L::kLatSlots;
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(&u_full[slot], (li / L::kLatSlots) & 1, kErrTimeoutTmaFull));
          if (!ok) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int b = 2 * k + bb;
            const uint64_t d_b = d_ring + (uint32_t)((slot * L::kLat + bb * L::kBlock) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              if (ptx::elect_one())
                ptx::mma_ts(scol, tmem + kColQ + 32 * b + 8 * ks, d_b + (uint32_t)((ks * 32) >> 4), idesc, 1u);
              __syncwarp();
            }
          }
          if (ptx::elect_one()) {
            ptx::mma_commit(&u_empty[slot]);
            if (k == L::kLatPerTile - 1) ptx::mma_commit(&s_full[jj & 1]);
          }
          __syncwarp();
        }
      }
      // nothing of ours may still run in the tensor core when TMEM is freed
      if (ptx::elect_one()) ptx::mma_commit(idle);
      __syncwarp();
      ptx::mbar_wait(idle, 0, kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax
    // the row sums and the partials' (m, l) are written after the previous kernel has finished
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int g = (int)(warp >> 2);                 // warpgroup: score tiles jj with jj % 2 == g
    const int qd = (int)(warp & 3);                 // TMEM lane quadrant
    const int h = qd * 32 + (int)lane;              // head within the group = TMEM lane
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const float sl2 = p.scale_log2;
    // reference max published by warpgroup x for its latest tile: 128 floats in staging slot x's tail
    auto m_slot = [&](int x) -> float* { return reinterpret_cast<float*>(smem + L::kOffM + x * 512); };
    float* end_l = reinterpret_cast<float*>(smem + L::kOffEndL);  // warpgroup 1's row sums at the end
    bool ok = true;
    float m_used = -INFINITY, l = 0.f;   // reference this warpgroup last used, and its row sum relative to it
    if (ntp > 0) {
      // q_abs row h, latent block b (columns 64b..) -> TMEM columns 32b.. (bf16 pairs); warpgroup g moves blocks 4g..4g+3
      const uint32_t v_base = ptx::map_peer(ptx::smem_u32(smem), 1);
#pragma unroll 1
      for (int pc = 2 * g; ok && pc < 2 * g + 2; ++pc) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&q_piece[pc], 0, kErrTimeoutTmaFull));
        if (!ok) break;
#pragma unroll 1
        for (int b = 2 * pc; b < 2 * pc + 2; ++b) {
          const uint8_t* src = smem + L::kOffQ + b * L::kBlock + h * 128;
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = *reinterpret_cast<const uint4*>(src + ((v ^ (h & 7)) << 4));
            r[4 * v] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
          }
          ptx::tmem_st32(tmem + lane_base + kColQ + 32 * b, r);
        }
        // the piece's shared memory has been read into registers: its slot may be refilled
        ptx::mbar_arrive(&q_free[pc]);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(q_ready);

      for (int jj = g; ok && jj < ntq; jj += 2) {
        const int sb = jj & 1;
        bool w = ptx::mbar_wait(&s_full[sb], (jj >> 1) & 1, kErrTimeoutMma);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t s_col = tmem + lane_base + kColS + sb * kTileQ;
        const int n_valid = (int)min64(kTileQ, u.j_end - (u.j_begin + (int64_t)jj * kTileQ));
        // S comes out of TMEM in one round trip (all 128 columns) and the buffer is handed back at
        // once, so that QK(jj+2) is not held up by the rest of this tile's softmax (the tensor
        // core, and with it the release of the ring slots, would otherwise wait on it)
        uint32_t a[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&a[32 * c]));
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::reg_fence32(&a[32 * c]);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&s_free[sb]);
        // row max of the raw scores over the valid keys (scale >= 0 commutes with max)
        float mx;
        {
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
          if (n_valid >= kTileQ) {
#pragma unroll
            for (int i = 0; i < 128; ++i) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(a[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i < n_valid) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(a[i]));
          }
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          mx *= sl2;
        }
        // the reference after tile jj-1 comes from the other warpgroup
        float m_prev = -INFINITY;
        if (jj > 0) {
          w = ptx::mbar_wait(&m_bar[g ^ 1], ((jj - 1) >> 1) & 1, kErrTimeoutSoftmax);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          m_prev = m_slot(g ^ 1)[h];
        }
        const float m_new = mx > m_prev + kRescaleThreshold ? mx : m_prev;
        m_slot(g)[h] = m_new;
        ptx::mbar_arrive(&m_bar[g]);
        const float f = (jj == 0 || m_new == m_prev) ? 1.f : fast_exp2(m_prev - m_new);
        if (m_used != m_new) {
          l = m_used == -INFINITY ? 0.f : l * fast_exp2(m_used - m_new);
          m_used = m_new;
        }
        // P = 2^(s * scale * log2(e) - m) as bf16, in two 64-key P tiles; keys past the end weigh
        // exactly 0.  Both P tiles are computed before the wait for the other warpgroup's P: only
        // the staging writes and copies are ordered between warpgroups, not the exponentials.
        const int nh = n_valid > kTileN ? 2 : 1;
        uint32_t pk[2][32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float ps0 = 0.f, ps1 = 0.f;
          if (kTileN * (half + 1) <= n_valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float e0 = fast_exp2(fmaf(__uint_as_float(a[64 * half + 2 * i]), sl2, -m_new));
              const float e1 = fast_exp2(fmaf(__uint_as_float(a[64 * half + 2 * i + 1]), sl2, -m_new));
              ps0 += e0;
              ps1 += e1;
              pk[half][i] = ptx::pack_bf16x2(e0, e1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int k = kTileN * half + 2 * i;
              float e0 = fast_exp2(fmaf(__uint_as_float(a[64 * half + 2 * i]), sl2, -m_new));
              float e1 = fast_exp2(fmaf(__uint_as_float(a[64 * half + 2 * i + 1]), sl2, -m_new));
              if (k >= n_valid) e0 = 0.f;
              if (k + 1 >= n_valid) e1 = 0.f;
              ps0 += e0;
              ps1 += e1;
              pk[half][i] = ptx::pack_bf16x2(e0, e1);
            }
          }
          l += ps0 + ps1;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half >= nh) break;
          const int t = 2 * jj + half, vs = t & 3;
          // P tiles reach the value CTA's slots strictly in order: the other warpgroup stored
          // those of score tile jj-1 first (and its copies have read the staging slot).  (It hands
          // over the reference max before its P, so without this a warpgroup could wait on a P slot
          // barrier two phases ahead, which a parity wait cannot tell from the phase before.)  The
          // value CTA's P slot vs is free once P V of tile t-4 finished.
          w = true;
          if (half == 0 && jj > 0) w = ptx::mbar_wait(&p_sent[g ^ 1], ((jj - 1) >> 1) & 1, kErrTimeoutSoftmax);
          if (t >= 4) w = w && ptx::mbar_wait<true>(&p_free[vs], ((t - 4) >> 2) & 1, kErrTimeoutPeer);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          // row h of the K-major P tile (128-byte swizzle) and the row's factor into the staging slot,
          // then this warp's 32 rows and factors to the value CTA's P slot vs (two bulk copies)
          uint8_t* stg = smem + L::kOffStaging;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stg + h * 128 + ((c ^ (h & 7)) << 4)) =
                make_uint4(pk[half][4 * c], pk[half][4 * c + 1], pk[half][4 * c + 2], pk[half][4 * c + 3]);
          reinterpret_cast<float*>(stg + ValueLayout::kOffF)[h] = half == 0 ? f : 1.f;
          ptx::fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            const uint32_t dst = v_base + ValueLayout::kOffSlots + (uint32_t)vs * ValueLayout::kSlot;
            const uint32_t vbar = v_base + ValueLayout::kOffBars + 8 * (bar::kPFull + vs);
            ptx::bulk_copy_to_peer(dst + qd * 4096, ptx::smem_u32(stg) + qd * 4096, 4096, vbar);
            ptx::bulk_copy_to_peer(dst + ValueLayout::kOffF + qd * 128, ptx::smem_u32(stg) + ValueLayout::kOffF + qd * 128,
                                   128, vbar);
            ptx::bulk_commit_group();
            // these rows of the staging slot are written again (the next half, or the other
            // warpgroup's next tile) only after the copies have read them
            ptx::bulk_wait_read_all();
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) ptx::mbar_arrive(&p_sent[g]);
      }
      // the row's final (m, l): both warpgroups' sums taken to the last reference
      // (warpgroup 1's last reference is the last one it published; it has none with one tile)
      if (g == 1) {
        end_l[h] = l;
        ptx::mbar_arrive(end_bar);
      } else if (ok) {
        const bool w = ptx::mbar_wait(end_bar, 0, kErrTimeoutSoftmax);
        if (__all_sync(0xffffffffu, w)) {
          const float l1 = end_l[h], m1 = ntq > 1 ? m_slot(1)[h] : -INFINITY;
          const float m_fin = fmaxf(m_used, m1);
          const float lt = l * fast_exp2(m_used - m_fin) + (m1 == -INFINITY ? 0.f : l1 * fast_exp2(m1 - m_fin));
          if (p.partials) {
            const int64_t slot = ((int64_t)u.sp * p.n_q + u.row) * p.heads + head0 + h;
            reinterpret_cast<float2*>(p.part_ml)[slot] = make_float2(m_fin, lt);
          }
          ptx::st_async_b32(v_base + ValueLayout::kOffL + 4 * h, v_base + ValueLayout::kOffBars + 8 * bar::kLFull,
                            __float_as_uint(lt));
        }
      }
    } else if (p.partials && g == 0) {
      // a split with no key contributes nothing to the merge
      const int64_t slot = ((int64_t)u.sp * p.n_q + u.row) * p.heads + head0 + h;
      reinterpret_cast<float2*>(p.part_ml)[slot] = make_float2(-INFINITY, 0.f);
    }
  }
}

// ---------------------------------------------------------------- value CTA
// Value CTA epilogue of one warp: rows 32qd.. (TMEM lanes) and latent columns 256c..256c+255 of O,
// scaled by inv, as bf16. TMEM is read 128 columns per round trip; each 64-column piece fills a
// 32-row x 128-byte box in shared memory (buf, 16 KB, 1024-byte aligned, 128-byte swizzle:
// conflict-free row writes) that leaves in its own tensor store at (0, y0, z0 + box) of the output
// map (whose third axis steps through 64-column blocks); the stores of the first two boxes overlap
// the second TMEM round trip. Returns once the boxes have been read out.
__device__ __forceinline__ void store_o_tma(uint8_t* buf, uint32_t t_base, uint32_t lane, float inv,
                                            const CUtensorMap* tmap_out, int32_t y0, int32_t z0) {
#pragma unroll 1
  for (int pr = 0; pr < 2; ++pr) {
    uint32_t r[128];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      ptx::tmem_ld32(t_base + 128 * pr + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * i]));
    ptx::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 4; ++i) ptx::reg_fence32(&r[32 * i]);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint8_t* box = buf + (2 * pr + k) * 4096;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t* x = &r[64 * k + 8 * j];
        *reinterpret_cast<uint4*>(box + lane * 128 + (((uint32_t)j ^ (lane & 7u)) << 4)) =
            make_uint4(ptx::pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                       ptx::pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                       ptx::pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                       ptx::pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
      }
    }
    ptx::fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      ptx::tma_store_3d(tmap_out, buf + (2 * pr) * 4096, 0, y0, z0 + 2 * pr);
      ptx::tma_store_3d(tmap_out, buf + (2 * pr + 1) * 4096, 0, y0, z0 + 2 * pr + 1);
      ptx::bulk_commit_group();
    }
    __syncwarp();
  }
  if (lane == 0) ptx::bulk_wait_read_all();
  __syncwarp();
}

template <bool kPaged>
__device__ __forceinline__ void value_role(uint8_t* smem, uint32_t tmem, const UnitRange& u, const AttnParams& p,
                                           const CUtensorMap* tmap_kv, const CUtensorMap* tmap_out) {
  using L = ValueLayout;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  uint64_t* v_full = bars + bar::kVFull;      // [2] kv tile landed
  uint64_t* v_empty = bars + bar::kVEmpty;    // [2] kv tile read by the tensor core
  uint64_t* p_full = bars + bar::kPFull;      // [4] P and factors of a tile landed (bulk copies from the score CTA)
  uint64_t* pv_go = bars + bar::kPvGo;        // [4] factors applied, tail cleared: P V may run (128 arrivals)
  uint64_t* p_done = bars + bar::kPDone;      // [4] P V product of this slot finished
  uint64_t* o_final = bars + bar::kOFinal;    // the last P V product finished
  uint64_t* l_full = bars + bar::kLFull;      // the row sums landed
  uint64_t* idle = bars + bar::kValueIdle;
  const uint32_t warp = ptx::warp_id(), lane = ptx::lane_id();
  const int nt = u.nt;

  if (warp == kProducerWarp) {
    // ============================================================ producer
    int issued = 0;
    if (nt > 0) {
      if (ptx::elect_one()) {
        ptx::prefetch_tmap(tmap_kv);
        ptx::prefetch_tmap(tmap_out);
      }
      __syncwarp();
      // The value tiles are the same rows the score CTA is loading: requested together they cost
      // HBM one read, and the first P V product need not wait for a load after the first P.  This
      // warp reads only the cache and writes no global memory: with p.early_cache (the previous
      // kernel does not write the cache) it never waits for the previous kernel, so the first
      // stages are requested at once and the first score tile finds its rows in L2.
      if (!p.early_cache) ptx::griddep_wait();
      CacheRows<kPaged> cache;
      cache.init(p, u, lane);
      for (int j = 0; j < nt; ++j) {
        const int st = j % L::kStages;
        const bool w = ptx::mbar_wait(&v_empty[st], ((j / L::kStages) & 1) ^ 1, kErrTimeoutStageFree);
        if (!__all_sync(0xffffffffu, w)) break;
        const int key = cache.row(u.j_begin + (int64_t)j * kTileN, u.j_end, lane);
        if (ptx::elect_one()) {
          ptx::mbar_arrive_expect_tx(&v_full[st], L::kStage);
          // one copy for the whole tile: eight 64-column blocks of 64 keys (the map's third axis
          // steps through the latent blocks), laid out block after block
          ptx::tma_load_3d(smem + st * L::kStage, tmap_kv, &v_full[st], 0, key, 0);
        }
        __syncwarp();
        issued = j + 1;
      }
      for (int j = (issued > L::kStages ? issued - L::kStages : 0); j < issued; ++j)
        ptx::mbar_wait(&v_full[j % L::kStages], (j / L::kStages) & 1, kErrTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ============================================================ MMA issuer
    // Two streams: P V of tile pv once its kv tile landed and its P was
    // released, and handing P slot fw back to the score CTA once P V of tile
    // fw finished (only for tiles the score CTA still waits on).
    if (nt > 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 256, false, true);
      const uint64_t d_p0 = ptx::smem_desc(ptx::smem_u32(smem + L::kOffSlots), 16, 1024, ptx::kSwizzle128);
      const uint64_t d_v0 = ptx::smem_desc(ptx::smem_u32(smem), L::kKvBox, 1024, ptx::kSwizzle128);
      const uint32_t score_free0 = ptx::map_peer(ptx::smem_u32(smem + ScoreLayout::kOffBars + 8 * bar::kPFree), 0);
      constexpr int kS = L::kPSlots;
      bool ok = true;
      int pv = 0, fw = 0;
      uint64_t t_last = global_timer_ns();
      while (ok && (pv < nt || fw < nt - kS)) {
        bool progressed = false;
        bool go = fw < nt - kS && fw < pv && ptx::mbar_test(&p_done[fw % kS], (fw / kS) & 1);
        if (__shfl_sync(0xffffffffu, go, 0)) {
          if (lane == 0) ptx::mbar_arrive_cluster_relaxed_addr(score_free0 + 8 * (fw % kS));
          __syncwarp();
          ++fw;
          progressed = true;
        }
        go = pv < nt && ptx::mbar_test(&v_full[pv % L::kStages], (pv / L::kStages) & 1) &&
             ptx::mbar_test(&pv_go[pv % kS], (pv / kS) & 1);
        if (__shfl_sync(0xffffffffu, go, 0)) {
          ptx::tc_fence_after();
          const uint32_t so = (uint32_t)((pv % L::kStages) * L::kStage) >> 4;
          const uint32_t po = (uint32_t)((pv % kS) * L::kSlot) >> 4;
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int ks = 0; ks < kTileN / 16; ++ks) {
              if (ptx::elect_one())
                ptx::mma_ss(tmem + 256 * n, d_p0 + po + (uint32_t)((ks * 32) >> 4),
                            d_v0 + so + (uint32_t)((n * 4 * L::kKvBox + ks * 2048) >> 4), idesc,
                            (pv > 0 || ks > 0) ? 1u : 0u);
              __syncwarp();
            }
          if (ptx::elect_one()) {
            ptx::mma_commit(&v_empty[pv % L::kStages]);
            ptx::mma_commit(&p_done[pv % kS]);
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
          const bool late = global_timer_ns() - t_last > kWaitLimitNs;
          if (__shfl_sync(0xffffffffu, late, 0)) {
            if (lane == 0) raise_error(pv < nt ? kErrTimeoutPeer : kErrTimeoutMma);
            ok = false;
          }
        }
      }
      if (ptx::elect_one()) ptx::mma_commit(idle);
      __syncwarp();
      ptx::mbar_wait(idle, 0, kErrTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ============================================================ warps 0-7
    // the epilogue's output is written after the previous kernel has finished
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int qd = (int)(warp & 3);
    const int h = qd * 32 + (int)lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    bool ok = true;
    if (nt > 0 && warp < 4) {
      // per tile: apply the row factors to O (rare), clear the tail rows, release P V
      if (threadIdx.x == 0) ptx::mbar_arrive_expect_tx(l_full, 512);
      constexpr int kS = L::kPSlots;
      for (int j = 0; j < nt; ++j) {
        const int s = j % kS;
        if (threadIdx.x == 0) ptx::mbar_arrive_expect_tx(&p_full[s], L::kP + 512);   // 4 x (4 KB + 128 B)
        bool w = ptx::mbar_wait<true>(&p_full[s], (j / kS) & 1, kErrTimeoutPeer);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        const float f = reinterpret_cast<const float*>(smem + L::kOffSlots + s * L::kSlot + L::kOffF)[h];
        if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
          // O holds the products of tiles < j relative to the old reference: scale it
          w = ptx::mbar_wait(&p_done[(j - 1) % kS], ((j - 1) / kS) & 1, kErrTimeoutMma);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base + 32 * c, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
            ptx::tmem_st32(tmem + lane_base + 32 * c, r);
          }
          ptx::tmem_wait_st();
        }
        const int n_valid = (int)min64(kTileN, u.j_end - (u.j_begin + (int64_t)j * kTileN));
        if (n_valid < kTileN) {
          // keys past the end have P = 0, but 0 * NaN is NaN: clear their value rows
          w = ptx::mbar_wait(&v_full[j % L::kStages], (j / L::kStages) & 1, kErrTimeoutTmaFull);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          uint8_t* st = smem + (j % L::kStages) * L::kStage;
          const int rows = kTileN - n_valid;
          for (int idx = (int)threadIdx.x; idx < 8 * rows * 8; idx += 128) {
            const int bx = idx / (rows * 8), rem = idx % (rows * 8);
            *reinterpret_cast<uint4*>(st + bx * L::kKvBox + (n_valid + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          ptx::fence_async_smem();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&pv_go[s]);
      }
    }
    // ---- epilogue: warp (qd, c) stores rows 32qd.. and latent columns 256c..256c+255 as bf16,
    // either o_lat = O / l (one split) or the split's partial O (relative to its final reference)
    const int c = (int)(warp >> 2);

    if (nt == 0) {
      if (!p.partials) {
        uint4* dst = reinterpret_cast<uint4*>(p.o_lat + (u.row * p.heads + u.hg * 128 + h) * 512 + 256 * c);
        for (int v = 0; v < 32; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      }
    } else {
      bool w = __all_sync(0xffffffffu, ok);
      w = w && ptx::mbar_wait(o_final, 0, kErrTimeoutMma);
      w = w && ptx::mbar_wait<true>(l_full, 0, kErrTimeoutPeer);   // also before exit: it writes here
      if (__all_sync(0xffffffffu, w)) {
        ptx::tc_fence_after();
        const float inv = p.partials ? 1.f : 1.f / reinterpret_cast<const float*>(smem + L::kOffL)[h];
        const int64_t row0 = (p.partials ? ((int64_t)u.sp * p.n_q + u.row) * p.heads : u.row * p.heads) +
                             u.hg * 128 + 32 * qd;
        // the value stages are idle once the last P V product finished: 16 KB of boxes per warp
        store_o_tma(smem + warp * 16384, tmem + lane_base + 256 * c, lane, inv, tmap_out, (int32_t)row0, 4 * c);

      }
    }
  }
}

// ---------------------------------------------------------------- the kernel
// The work of one CTA of a pair on its unit (query row, 128-head group, split): set-up, then the
// score or the value role.  Returns the TMEM base, still allocated (attn_teardown frees it).
template <bool kPaged>
__device__ __forceinline__ uint32_t attn_unit(uint8_t* smem, const CUtensorMap* tmap_kv_score,
                                              const CUtensorMap* tmap_pe, const CUtensorMap* tmap_qpe,
                                              const CUtensorMap* tmap_kv_value, const CUtensorMap* tmap_qabs,
                                              const CUtensorMap* tmap_out, const AttnParams& p) {
  const uint32_t warp = ptx::warp_id();
  const uint32_t rank = ptx::cluster_rank();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (rank == 0 ? ScoreLayout::kOffBars : ValueLayout::kOffBars));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + bar::kTmemSlot);
  // the swizzled tiles need a 1024-byte aligned base (both CTAs see the same alignment)
  const bool aligned = (ptx::smem_u32(smem) & 1023u) == 0;

  if (threadIdx.x == 0) {
    if (rank == 0) {
      for (int s = 0; s < ScoreLayout::kLatSlots; ++s) {
        ptx::mbar_init(&bars[bar::kUFull + s], 1);
        ptx::mbar_init(&bars[bar::kUEmpty + s], 1);
      }
      for (int s = 0; s < ScoreLayout::kPeSlots; ++s) {
        ptx::mbar_init(&bars[bar::kPeFull + s], 1);
        ptx::mbar_init(&bars[bar::kPeEmpty + s], 1);
      }
      for (int s = 0; s < 2; ++s) {
        ptx::mbar_init(&bars[bar::kSFull + s], 1);
        ptx::mbar_init(&bars[bar::kSFree + s], 128);
        ptx::mbar_init(&bars[bar::kMBar + s], 128);
        ptx::mbar_init(&bars[bar::kPSent + s], 4);
      }
      for (int s = 0; s < ValueLayout::kPSlots; ++s) ptx::mbar_init(&bars[bar::kPFree + s], 1);
      ptx::mbar_init(&bars[bar::kQFull], 1);
      for (int k = 0; k < 4; ++k) {
        ptx::mbar_init(&bars[bar::kQPiece + k], 1);
        ptx::mbar_init(&bars[bar::kQFree + k], 128);
      }
      ptx::mbar_init(&bars[bar::kQReady], 256);
      ptx::mbar_init(&bars[bar::kEnd], 128);
      ptx::mbar_init(&bars[bar::kScoreIdle], 1);
    } else {
      for (int s = 0; s < ValueLayout::kStages; ++s) {
        ptx::mbar_init(&bars[bar::kVFull + s], 1);
        ptx::mbar_init(&bars[bar::kVEmpty + s], 1);
      }
      for (int s = 0; s < ValueLayout::kPSlots; ++s) {
        ptx::mbar_init(&bars[bar::kPFull + s], 1);
        ptx::mbar_init(&bars[bar::kPvGo + s], 128);
        ptx::mbar_init(&bars[bar::kPDone + s], 1);
      }
      ptx::mbar_init(&bars[bar::kOFinal], 1);
      ptx::mbar_init(&bars[bar::kLFull], 1);
      ptx::mbar_init(&bars[bar::kValueIdle], 1);
    }
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
  // Set-up above touches no global memory.  q_abs and q_pe may come from the previous kernel in
  // the stream, and the outputs may still be read by it: the warps that load q or write outputs
  // wait for it first (griddepcontrol.wait) in their roles; the MMA warps touch no global memory.
  // The unit's key range (cu_seqlens) is read before that wait, and with p.early_cache the value
  // CTA's producer starts its cache stream before it.
  UnitRange u = unit_range(p, blockIdx.x >> 1);
  if (!aligned) {
    if (threadIdx.x == 0) raise_error(kErrBadSchedule);
    u.nt = 0;
  }
  if (rank == 0)
    score_role<kPaged>(smem, tmem, u, p, tmap_kv_score, tmap_pe, tmap_qpe, tmap_qabs);
  else
    value_role<kPaged>(smem, tmem, u, p, tmap_kv_value, tmap_out);
  return tmem;
}

__device__ __forceinline__ void attn_teardown(uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if (ptx::warp_id() == kMmaWarp) ptx::tmem_dealloc(tmem, 512);
  ptx::cluster_sync();   // neither CTA's shared memory goes away while the partner may still write into it
}

// One cluster of two CTAs per work unit (query row, 128-head group, split).
// kPaged: the cache is read through a block table (one instance per cache kind).
template <bool kPaged>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    latent_attn_kernel(const __grid_constant__ CUtensorMap tmap_kv_score, const __grid_constant__ CUtensorMap tmap_pe,
                       const __grid_constant__ CUtensorMap tmap_qpe, const __grid_constant__ CUtensorMap tmap_kv_value,
                       const __grid_constant__ CUtensorMap tmap_qabs, const __grid_constant__ CUtensorMap tmap_out,
                       const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t tmem = attn_unit<kPaged>(smem, &tmap_kv_score, &tmap_pe, &tmap_qpe, &tmap_kv_value, &tmap_qabs,
                                          &tmap_out, p);
  attn_teardown(tmem);
}

// Merge split partials: o = sum_s 2^{m_s - M} O_s / sum_s 2^{m_s - M} l_s, M = max_s m_s,
// with O_s the bf16 partial of split s (relative to its reference m_s).
// Two warps per (row, head), four per block; lane i of warp k owns columns
// 256k + 8i .. +7.  A lane starts loading its columns of (up to) the first
// kMergeInFlight splits, then reads the (m, l) pair of split `lane` (one round
// trip; weights reach the other lanes by shuffle), so the two memory round trips
// overlap.  The kernel needs no shared memory: its blocks can be resident beside
// the attention CTAs and start as soon as the attention grid completes.  Splits
// with no key (m = -inf) get weight 0 and their (unwritten) partial is never used.
constexpr int kMergeInFlight = 16;
constexpr int kMergeThreads = 128;

__device__ __forceinline__ void merge_acc(float (&a)[8], float w, const uint4& x) {
  const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
    a[2 * i] = fmaf(w, f.x, a[2 * i]);
    a[2 * i + 1] = fmaf(w, f.y, a[2 * i + 1]);
  }
}

// The merge weights of one (row, head) as a warp computes them: lane s < 32 returns the weight
// 2^(m_s - M) of split s (0 for a split with no key); M = max_s m_s and inv = 1 / sum_s w_s l_s
// (0 when no split saw a key).  ml points at the (m, l) pair of split 0, split_stride pairs apart.
// Both consumers of the partials (merge_splits_kernel, merge_proj_kernel) use this, so they
// produce bit-identical o_lat rows.
__device__ __forceinline__ float merge_weights(const float2* ml, int64_t split_stride, int num_splits, int lane,
                                               float& M_out, float& inv_out) {
  const float2 mine = lane < num_splits ? __ldcg(ml + lane * split_stride) : make_float2(-INFINITY, 0.f);
  float M = mine.x;
  for (int s = lane + 32; s < num_splits; s += 32) M = fmaxf(M, __ldcg(ml + s * split_stride).x);
  M = warp_max(M);
  const float w_lane = mine.x == -INFINITY ? 0.f : exp2f(mine.x - M);
  float L = w_lane * mine.y;
  for (int s = lane + 32; s < num_splits; s += 32) {
    const float2 x = __ldcg(ml + s * split_stride);
    if (x.x != -INFINITY) L += exp2f(x.x - M) * x.y;
  }
  L = warp_sum(L);
  M_out = M;
  inv_out = L > 0.f ? 1.f / L : 0.f;
  return w_lane;
}

__global__ void __launch_bounds__(kMergeThreads) merge_splits_kernel(const __nv_bfloat16* __restrict__ part_o,
                                                                 const float* __restrict__ part_ml, int num_splits,
                                                                 int64_t n_q, int heads,
                                                                 __nv_bfloat16* __restrict__ o_lat) {
  // the next kernel may launch now: its set-up (and, for the output projection, its weight
  // stream) overlaps this kernel, and it waits for this grid before reading o_lat
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int64_t warp_g = (int64_t)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  const int64_t pair = warp_g >> 1;
  if (pair >= n_q * heads) return;   // warp-uniform
  const int lane = (int)(threadIdx.x & 31);
  const int64_t split_stride = n_q * heads;
  const uint4* src = reinterpret_cast<const uint4*>(part_o + pair * 512) + 32 * (warp_g & 1) + lane;
  const int64_t step = split_stride * 512 / 8;   // one split further, in 16-byte units
  uint4 v[kMergeInFlight];
#pragma unroll
  for (int s = 0; s < kMergeInFlight; ++s)
    if (s < num_splits) v[s] = __ldcg(src + s * step);
  const float2* ml = reinterpret_cast<const float2*>(part_ml) + pair;
  float M, inv;
  const float w_lane = merge_weights(ml, split_stride, num_splits, lane, M, inv);   // the weight of split `lane`
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = 0.f;
#pragma unroll
  for (int s = 0; s < kMergeInFlight; ++s)
    if (s < num_splits) {
      const float w = __shfl_sync(0xffffffffu, w_lane, s);
      if (w != 0.f) merge_acc(a, w, v[s]);
    }
  for (int s = kMergeInFlight; s < num_splits; ++s) {
    const float w = __shfl_sync(0xffffffffu, w_lane, s & 31);
    const float2 x = __ldcg(ml + s * split_stride);   // splits >= 32: not in a lane's register
    const float ws = s < 32 ? w : (x.x == -INFINITY ? 0.f : exp2f(x.x - M));
    if (ws != 0.f) merge_acc(a, ws, __ldcg(src + s * step));
  }
  uint4 o;
  o.x = ptx::pack_bf16x2(a[0] * inv, a[1] * inv);
  o.y = ptx::pack_bf16x2(a[2] * inv, a[3] * inv);
  o.z = ptx::pack_bf16x2(a[4] * inv, a[5] * inv);
  o.w = ptx::pack_bf16x2(a[6] * inv, a[7] * inv);
  reinterpret_cast<uint4*>(o_lat + pair * 512)[32 * (warp_g & 1) + lane] = o;
}

}  // namespace sm100
}  // namespace mla
