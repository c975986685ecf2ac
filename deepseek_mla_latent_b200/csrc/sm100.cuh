// sm100.cuh -- host side of the tensor-core (tcgen05) path for the
// DeepSeek-V3 head shapes: TMA descriptor encoding, launch shapes, split-t
// planning and the workspace layout.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "mla.h"
#include "sm100_attn.cuh"
#include "sm100_expand.cuh"
#include "sm100_fmha.cuh"
#include "sm100_merge_proj.cuh"
#include "sm100_decode_fused.cuh"
#include "sm100_proj.cuh"

namespace mla {
namespace sm100 {

inline bool supports(int H, int C, int Dn, int R, int Dv) {
  return C == 512 && R == 64 && Dn == 128 && Dv == 128 && H > 0 && H % 128 == 0 && H <= 128 * 64;
}

// ---------------------------------------------------------------- TMA maps --
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map (bf16 unless `dt` says otherwise): dims/strides innermost first, strides in bytes (rank-1 of them).
inline bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                     const uint32_t* box, CUtensorMapSwizzle swz,
                     CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides[i];
  return fn(m, dt, rank, const_cast<void*>(base), d, s, b, e,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Four-dimensional map without swizzle (bf16): dims/strides innermost first, strides in bytes.
inline bool make_map4(CUtensorMap* m, const void* base, const uint64_t* dims, const uint64_t* strides,
                      const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[4], s3[3];
  cuuint32_t b[4], e[4] = {1, 1, 1, 1};
  for (int i = 0; i < 4; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i < 3; ++i) s3[i] = strides[i];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), d, s3, b, e,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline mla_status_t last_launch() { return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Launch with programmatic stream serialization (pdl = true): the kernel may
// start its set-up while the previous kernel in the stream finishes; every
// kernel here waits (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
inline mla_status_t launch(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device); the
// call is host-side only, so it is also safe while a stream is being captured.
inline bool set_smem_once(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == kernel && d.second == dev) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
  done.emplace_back(kernel, dev);
  return true;
}
template <typename K>
inline bool set_smem(K kernel, size_t bytes) {
  return set_smem_once(reinterpret_cast<const void*>(kernel), bytes);
}

// --------------------------------------------------------------- projections
template <bool A_MN, int N_TILE, int STAGES>
inline mla_status_t launch_proj(const CUtensorMap& tw, const CUtensorMap& tx, dim3 grid, int k_chunks, int w_row_base,
                                int n_rows, void* out, int64_t out_row_stride, int out_head_stride,
                                cudaStream_t stream, bool pdl) {
  constexpr size_t smem = proj_smem_bytes<N_TILE, STAGES>();
  auto kern = proj_kernel<A_MN, N_TILE, STAGES>;
  if (!set_smem(kern, smem)) return MLA_ERR_CUDA;
  return launch(pdl, kern, grid, dim3(kProjThreads), smem, stream, tw, tx, k_chunks, w_row_base, 256, n_rows,
                static_cast<__nv_bfloat16*>(out), out_row_stride, out_head_stride);
}

// STAGES: the K ring depth; with few query rows the whole weight tile of a
// CTA is kept in flight (the projection is a weight stream at decode sizes).
template <bool A_MN, int MAX_STAGES>
inline mla_status_t dispatch_proj(const CUtensorMap& tw, const CUtensorMap& tx, int m_tiles, int H, int64_t n_rows,
                                  int k_chunks, int w_row_base, void* out, int64_t out_row_stride,
                                  int out_head_stride, cudaStream_t stream, bool pdl) {
  auto go = [&](auto tile) {
    constexpr int NT = decltype(tile)::value;
    constexpr int STAGES = NT <= 64 ? MAX_STAGES : (MAX_STAGES < 4 ? MAX_STAGES : 4);
    if ((n_rows + NT - 1) / NT > 65535 || H > 65535) return MLA_ERR_INVALID_ARG;   // grid's y and z axes
    dim3 grid(m_tiles, H, (unsigned)((n_rows + NT - 1) / NT));
    return launch_proj<A_MN, NT, STAGES>(tw, tx, grid, k_chunks, w_row_base, (int)n_rows, out, out_row_stride,
                                         out_head_stride, stream, pdl);
  };
  if (n_rows <= 16) return go(std::integral_constant<int, 16>{});
  if (n_rows <= 32) return go(std::integral_constant<int, 32>{});
  if (n_rows <= 64) return go(std::integral_constant<int, 64>{});
  if (n_rows <= 128) return go(std::integral_constant<int, 128>{});
  return go(std::integral_constant<int, 256>{});
}

inline mla_status_t absorb_q(const void* q, int64_t q_row_stride, const void* wkv_b, void* q_abs, int64_t n_rows,
                             int H, cudaStream_t stream) {
  if (n_rows >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  CUtensorMap tw, tx;
  const uint64_t wd[2] = {512, (uint64_t)H * 256}, ws[1] = {1024};
  const uint32_t wb[2] = {64, 64};   // 64 latent columns x 64 key rows (M-major A)
  const uint64_t xd[3] = {192, (uint64_t)H, (uint64_t)n_rows}, xs[2] = {384, (uint64_t)q_row_stride * 2};
  const uint32_t xb[3] = {64, 1, 0};
  uint32_t box[3] = {xb[0], xb[1], (uint32_t)(n_rows <= 16 ? 16 : n_rows <= 32 ? 32 : n_rows <= 64 ? 64 : n_rows <= 128 ? 128 : 256)};
  if (!make_map(&tw, wkv_b, 2, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  if (!make_map(&tx, q, 3, xd, xs, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  // the first kernel of a step: its weight copies (wkv_b is never written by the kernels of a step)
  // start before the wait for the previous kernel, so they overlap the previous layer's tail
  return dispatch_proj<true, 2>(tw, tx, 4, H, n_rows, 2, 0, q_abs, (int64_t)H * 512, 512, stream, true);
}

inline mla_status_t out_proj(const void* o_lat, const void* wkv_b, void* out, int64_t n_rows, int H,
                             cudaStream_t stream) {
  if (n_rows >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  CUtensorMap tw, tx;
  const uint64_t wd[2] = {512, (uint64_t)H * 256}, ws[1] = {1024};
  const uint32_t wb[2] = {64, 128};  // 64 latent columns x 128 value rows (K-major A)
  const uint64_t xd[3] = {512, (uint64_t)H, (uint64_t)n_rows}, xs[2] = {1024, (uint64_t)H * 1024};
  uint32_t box[3] = {64, 1, (uint32_t)(n_rows <= 16 ? 16 : n_rows <= 32 ? 32 : n_rows <= 64 ? 64 : n_rows <= 128 ? 128 : 256)};
  if (!make_map(&tw, wkv_b, 2, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  if (!make_map(&tx, o_lat, 3, xd, xs, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  return dispatch_proj<false, 8>(tw, tx, 1, H, n_rows, 8, 128, out, (int64_t)H * 128, 128, stream, true);
}

// ----------------------------------------------------------------- attention
inline int prefill_splits() { return 1; }

// Split-t plan for decode: enough (row, head group, split) units to give
// each CTA pair of the GPU one, splits never shorter than one 128-key score tile.
inline int auto_decode_splits(int batch, int H, int64_t max_seqlen_k, int sms) {
  if (batch <= 0) return 1;
  const int64_t pairs = sms / 2;
  const int64_t rows = (int64_t)batch * (H / 128);
  int64_t s = pairs / rows;
  const int64_t max_tiles = (max_seqlen_k + kTileQ - 1) / kTileQ;
  if (s > max_tiles) s = max_tiles;
  if (s > 256) s = 256;
  if (s < 1) return 1;
  // splits are whole score tiles: with `per` keys per split the longest sequence fills only
  // ceil(t / per) of them, and a unit with no key would only hold a CTA pair
  const int64_t per = ((max_seqlen_k + s - 1) / s + kTileQ - 1) / kTileQ * kTileQ;
  const int64_t used = (max_seqlen_k + per - 1) / per;
  return (int)(used < s ? used : s);
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t workspace_bytes(int H, int64_t n_q, int splits, bool partials = false) {
  if (splits <= 1 && !partials) return 0;
  // bf16 partial O per (split, row, head) + fp32 (reference max, row sum)
  return align256((size_t)splits * n_q * H * 512 * 2) + align256((size_t)splits * n_q * H * 2 * sizeof(float));
}

// Split partials in the workspace: bf16 O [splits, n_q, H, 512], then fp32 (m, l) [splits, n_q, H, 2].
inline size_t partial_ml_offset(int H, int64_t n_q, int splits) {
  return align256((size_t)splits * n_q * H * 512 * 2);
}

// Addressing of a paged cache: sequence b holds seqlens[b] keys, key j in row
// table[b * stride + j / page] * page + j % page.  table == nullptr: packed cache (cu_k).
struct PagedKv {
  const int32_t* seqlens = nullptr;
  const int32_t* table = nullptr;
  int64_t stride = 0;
  int page = 0;
};

// The tensor maps and parameters of the latent attention kernel for one call.
struct AttnLaunch {
  CUtensorMap tkv_s, tpe, tqpe, tkv_v, tqa, tout;
  AttnParams p;
  int64_t units = 0;
  __nv_bfloat16* part_o = nullptr;
};

inline mla_status_t prepare_attention(AttnLaunch& L, const void* q_abs, const void* q, int64_t q_row_stride,
                                      const void* kv, const void* pe, int64_t kv_rows, const int32_t* cu_q,
                                      const int32_t* cu_k, int batch, int64_t n_q, int H, int splits, float scale,
                                      void* o_lat, void* ws, const PagedKv& paged, bool partials,
                                      bool early_cache = true) {
  CUtensorMap &tkv_s = L.tkv_s, &tpe = L.tpe, &tqpe = L.tqpe, &tkv_v = L.tkv_v, &tqa = L.tqa, &tout = L.tout;
  AttnParams& p = L.p;
  if (paged.table && (paged.page <= 0 || paged.page % kTileN != 0 || !paged.seqlens || paged.stride < 0))
    return MLA_ERR_INVALID_ARG;
  // pages of 64 * odd keys: the score CTA copies 64 keys at a time
  const uint32_t score_rows = paged.table && paged.page % kTileQ != 0 ? kTileN : kTileQ;
  if (kv_rows >= (1LL << 31) || n_q >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  const int64_t units = n_q * (H / 128) * splits;
  L.units = units;
  if (units == 0) return MLA_OK;
  if (2 * units >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  if ((uint64_t)n_q * H * (uint64_t)splits >= (1ULL << 31)) return MLA_ERR_INVALID_ARG;
  // kv_rows may be 0 (every sequence empty); the maps still need one row.
  const uint64_t rows = kv_rows > 0 ? (uint64_t)kv_rows : 1;
  const void* kv_base = kv_rows > 0 ? kv : q_abs;   // any valid 16-byte aligned address for an unused map
  const void* pe_base = kv_rows > 0 ? pe : q_abs;
  {
    // the cache as [8 latent blocks][rows][64 columns] (block stride 128 bytes): the score CTA
    // copies two 64-column blocks of 128 keys at a time (one block of 64 keys with 64 * odd
    // pages), the value CTA a whole 64-key tile (eight blocks) at a time
    const uint64_t d3[3] = {64, rows, 8}, st3[2] = {1024, 128};
    const uint32_t bs[3] = {64, score_rows, score_rows == kTileQ ? 2u : 1u};
    if (!make_map(&tkv_s, kv_base, 3, d3, st3, bs, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    const uint32_t bv[3] = {64, (uint32_t)kTileN, 8};
    if (!make_map(&tkv_v, kv_base, 3, d3, st3, bv, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t d[2] = {64, rows}, st[1] = {128};
    const uint32_t b[2] = {64, score_rows};           // 64 rotary columns x 128 (or 64) keys
    if (!make_map(&tpe, pe_base, 2, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    // q viewed as [n_q, H, 192]; the box is the rotary part (columns 128..191) of 128 heads of one row
    const uint64_t d[3] = {192, (uint64_t)H, (uint64_t)n_q}, st[2] = {384, (uint64_t)q_row_stride * 2};
    const uint32_t b[3] = {64, 128, 1};
    if (!make_map(&tqpe, q, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    // q_abs viewed as [8 latent blocks][n_q * H rows][64 columns] (block stride 128 bytes): one box
    // is two 64-column blocks of a unit's 128 heads (32 KB)
    const uint64_t d[3] = {64, (uint64_t)n_q * H, 8}, st[2] = {1024, 128};
    const uint32_t b[3] = {64, 128, 2};
    if (!make_map(&tqa, q_abs, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  p.q_abs = static_cast<const __nv_bfloat16*>(q_abs);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.seqlens_k = paged.seqlens;
  p.block_table = paged.table;
  p.bt_stride = paged.stride;
  p.page_size = paged.page;
  p.score_copy_rows = (int)score_rows;
  p.batch = batch;
  p.heads = H;
  p.head_groups = H / 128;
  p.num_splits = splits;
  p.partials = (splits > 1 || partials) ? 1 : 0;
  p.early_cache = early_cache ? 1 : 0;
  p.kv_rows = kv_rows;
  p.n_q = n_q;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_lat = static_cast<__nv_bfloat16*>(o_lat);
  p.part_ml = nullptr;

  __nv_bfloat16* part_o = nullptr;
  if (p.partials) {
    part_o = static_cast<__nv_bfloat16*>(ws);
    p.part_ml = reinterpret_cast<float*>(static_cast<char*>(ws) + partial_ml_offset(H, n_q, splits));
  }
  p.out = p.partials ? part_o : static_cast<__nv_bfloat16*>(o_lat);
  {
    // the epilogue's output rows (o_lat, or the bf16 split partials) as [8 latent blocks][rows][64]:
    // boxes of 32 heads x 64 columns (an epilogue warp writes four of them)
    const uint64_t d[3] = {64, (uint64_t)(p.partials ? splits : 1) * n_q * H, 8}, st[2] = {1024, 128};
    const uint32_t b[3] = {64, 32, 1};
    if (!make_map(&tout, p.out, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  L.part_o = part_o;
  return MLA_OK;
}

// The split merge alone: o_lat [n_q, H, 512] from split partials (part_o bf16 [splits, n_q, H, 512],
// part_ml fp32 [splits, n_q, H, 2]).
inline mla_status_t merge_partials(const void* part_o, const void* part_ml, int splits, int64_t n_q, int H,
                                   void* o_lat, cudaStream_t stream) {
  if (splits < 1 || n_q >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  const int64_t pairs_per_block = kMergeThreads / 64;   // two warps per (row, head)
  const int64_t merge_blocks = (n_q * H + pairs_per_block - 1) / pairs_per_block;
  if (merge_blocks >= (1LL << 31)) return MLA_ERR_INVALID_ARG;   // one grid dimension
  return launch(true, merge_splits_kernel, dim3((unsigned)merge_blocks), dim3(kMergeThreads), 0, stream,
                static_cast<const __nv_bfloat16*>(part_o), static_cast<const float*>(part_ml), splits, n_q, H,
                static_cast<__nv_bfloat16*>(o_lat));
}

// merge = false (split runs only): leave the partials in the workspace for merge_out_proj
// instead of merging them into o_lat.  partials = true: write the partial form (also for one
// split) and never merge; o_lat is not used.
inline mla_status_t attention(const void* q_abs, const void* q, int64_t q_row_stride, const void* kv, const void* pe,
                              int64_t kv_rows, const int32_t* cu_q, const int32_t* cu_k, int batch, int64_t n_q,
                              int H, int splits, float scale, void* o_lat, void* ws, cudaStream_t stream,
                              bool merge = true, const PagedKv& paged = PagedKv{}, bool partials = false,
                              bool early_cache = true) {
  AttnLaunch L;
  mla_status_t st = prepare_attention(L, q_abs, q, q_row_stride, kv, pe, kv_rows, cu_q, cu_k, batch, n_q, H, splits,
                                      scale, o_lat, ws, paged, partials, early_cache);
  if (st != MLA_OK || L.units == 0) return st;
  const AttnParams& p = L.p;
  auto kern = paged.table ? latent_attn_kernel<true> : latent_attn_kernel<false>;
  if (!set_smem(kern, kAttnSmem)) return MLA_ERR_CUDA;
  st = launch(true, kern, dim3((unsigned)(2 * L.units)), dim3(kAttnThreads), kAttnSmem, stream, L.tkv_s, L.tpe,
              L.tqpe, L.tkv_v, L.tqa, L.tout, p);
  if (st != MLA_OK || splits <= 1 || !merge || partials) return st;
  return merge_partials(L.part_o, p.part_ml, splits, n_q, H, o_lat, stream);
}

// Decode attention, split merge and output projection in one kernel (decode_fused_kernel).
// ws: the attention's split partials, then 256 bytes of control words (zero before the call,
// left zero after it).  Needs splits >= 2 and no more CTAs (2 per unit) than SMs.
inline bool fused_fits(int batch, int H, int splits, int sms) {
  return splits >= 2 && splits <= kMergeMaxSplitsFused && (int64_t)batch * (H / 128) * splits * 2 <= sms &&
         (int64_t)(batch < kMpRows ? batch : kMpRows) * splits <= FusedTailSmem::kMaxRowSplits;
}

inline mla_status_t decode_fused(const void* q_abs, const void* q, int64_t q_row_stride, const void* kv,
                                 const void* pe, int64_t kv_rows, const int32_t* cu_k, int batch, int H, int splits,
                                 float scale, const void* wkv_b, void* out, void* ws, uint32_t* ctrl,
                                 cudaStream_t stream) {
  AttnLaunch L;
  mla_status_t st = prepare_attention(L, q_abs, q, q_row_stride, kv, pe, kv_rows, nullptr, cu_k, batch, batch, H,
                                      splits, scale, nullptr, ws, PagedKv{}, /*partials=*/true);
  if (st != MLA_OK || L.units == 0) return st;
  CUtensorMap tw;
  {
    // wkv_b as [8 latent blocks][H * 256 rows][64 columns]: one box is a head's 128 value rows
    const uint64_t d[3] = {64, (uint64_t)H * 256, 8}, stw[2] = {1024, 128};
    const uint32_t b[3] = {64, 128, 8};
    if (!make_map(&tw, wkv_b, 3, d, stw, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  FusedParams f;
  f.part_rows = batch < kMpRows ? batch : kMpRows;
  if ((int64_t)f.part_rows * splits > FusedTailSmem::kMaxRowSplits) return MLA_ERR_INVALID_ARG;
  {
    // the split partials as [splits][n_q][H][512]: a box is 256 columns of one head for R rows and
    // every split
    const uint64_t d[4] = {512, (uint64_t)H, (uint64_t)batch, (uint64_t)splits};
    const uint64_t st[3] = {1024, (uint64_t)H * 1024, (uint64_t)batch * H * 1024};
    const uint32_t b[4] = {256, 1, (uint32_t)f.part_rows, (uint32_t)splits};
    if (!make_map4(&f.tmap_part, L.part_o, d, st, b)) return MLA_ERR_CUDA;
  }
  f.ctrl = ctrl;
  f.row_tiles = (batch + kMpRows - 1) / kMpRows;
  f.n_items = H * f.row_tiles;
  f.part_o = L.part_o;
  f.part_ml = L.p.part_ml;
  f.num_splits = splits;
  f.n_q = batch;
  f.heads = H;
  f.out = static_cast<__nv_bfloat16*>(out);
  if (!set_smem(decode_fused_kernel, kAttnSmem)) return MLA_ERR_CUDA;
  return launch(true, decode_fused_kernel, dim3((unsigned)(2 * L.units)), dim3(kAttnThreads), kAttnSmem, stream,
                L.tkv_s, L.tpe, L.tqpe, L.tkv_v, L.tqa, L.tout, tw, L.p, f);
}

// The output projection with the split merge fused in: out [n_q, H, 128] from split partials
// (part_o bf16 [splits, n_q, H, 512], part_ml fp32 [splits, n_q, H, 2]).
inline mla_status_t merge_partials_out(const void* part_o, const void* part_ml, int splits, int64_t n_q, int H,
                                       const void* wkv_b, void* out, cudaStream_t stream) {
  if (splits < 1 || splits > kMpMaxSplits || n_q >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  if ((n_q + kMpRows - 1) / kMpRows > 65535) return MLA_ERR_INVALID_ARG;   // row tiles on the grid's y axis
  CUtensorMap tw;
  // wkv_b as [8 latent blocks][H * 256 rows][64 columns]: one box is a head's 128 value rows, all
  // eight 64-column K chunks (128 KB, K-major A chunks 16 KB apart)
  const uint64_t wd[3] = {64, (uint64_t)H * 256, 8}, wst[2] = {1024, 128};
  const uint32_t wb[3] = {64, 128, 8};
  if (!make_map(&tw, wkv_b, 3, wd, wst, wb, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  constexpr size_t smem = merge_proj_smem_bytes();
  if (!set_smem(merge_proj_kernel, smem)) return MLA_ERR_CUDA;
  return launch(true, merge_proj_kernel, dim3((unsigned)H, (unsigned)((n_q + kMpRows - 1) / kMpRows)),
                dim3(kMergeProjThreads), smem, stream, tw, static_cast<const __nv_bfloat16*>(part_o),
                static_cast<const float*>(part_ml), splits, (int)n_q, H, static_cast<__nv_bfloat16*>(out));
}

// The same for the partials an attention(..., merge = false) call left in ws.
inline mla_status_t merge_out_proj(const void* ws, int splits, int64_t n_q, int H, const void* wkv_b, void* out,
                                   cudaStream_t stream) {
  if (splits < 2) return MLA_ERR_INVALID_ARG;
  return merge_partials_out(ws, static_cast<const char*>(ws) + partial_ml_offset(H, n_q, splits), splits, n_q, H,
                            wkv_b, out, stream);
}

// Latent KV expansion: K_nope and V [batch, H, seq_len, 128] from kv_c [batch * seq_len, 512].
inline mla_status_t expand_kv(const void* kv_c, const void* gamma, float eps, const void* wkv_b, int64_t batch,
                              int64_t seq_len, int H, void* k_nope, void* v, int sms, cudaStream_t stream) {
  const int64_t n_tokens = batch * seq_len;
  if (n_tokens == 0) return MLA_OK;
  if (n_tokens >= (1LL << 31) || (int64_t)H * 256 >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  CUtensorMap tx, tw;
  {
    // kv_c as [8 latent blocks][tokens][64 columns] (block stride 128 bytes): one box is a
    // 128-token tile, all eight blocks
    const uint64_t d[3] = {64, (uint64_t)n_tokens, 8}, st[2] = {1024, 128};
    const uint32_t b[3] = {64, 128, 8};
    if (!make_map(&tx, kv_c, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t d[2] = {512, (uint64_t)H * 256}, st[1] = {1024};
    const uint32_t b[2] = {64, 256};   // 64 latent columns of one head's 256 rows
    if (!make_map(&tw, wkv_b, 2, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  ExpandParams p;
  p.gamma = static_cast<const __nv_bfloat16*>(gamma);
  p.eps = eps;
  p.n_tokens = n_tokens;
  p.seq_len = seq_len;
  p.heads = H;
  p.n_items = (n_tokens + 127) / 128 * H;
  p.k_nope = static_cast<__nv_bfloat16*>(k_nope);
  p.v = static_cast<__nv_bfloat16*>(v);
  p.vec32 = ((reinterpret_cast<uintptr_t>(k_nope) | reinterpret_cast<uintptr_t>(v)) & 31u) == 0;
  const int64_t grid = p.n_items < sms ? p.n_items : sms;
  constexpr size_t smem = expand_smem_bytes();
  if (!set_smem(expand_kernel, smem)) return MLA_ERR_CUDA;
  return launch(false, expand_kernel, dim3((unsigned)grid), dim3(kExThreads), smem, stream, tx, tw, p);
}

// Per-head attention over expanded keys and values (the naive path of a chunked prefill):
// out [n_q, H, 128] from q [n_q, H, 192] (row stride q_row_stride elements), K_nope and V
// [H, kv_rows, 128] and pe [kv_rows, 64].
inline mla_status_t attention_expanded(const void* q, int64_t q_row_stride, const void* k_nope, const void* v,
                                       const void* pe, int64_t kv_rows, const int32_t* cu_q, const int32_t* cu_k,
                                       int batch, int64_t n_q, int64_t max_seqlen_q, int H, float scale, void* out,
                                       int sms, cudaStream_t stream) {
  if (n_q >= (1LL << 31) || kv_rows >= (1LL << 31) || max_seqlen_q >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  const int64_t q_pairs = (max_seqlen_q + 2 * kFaTile - 1) / (2 * kFaTile);
  const int64_t units = (int64_t)batch * H * q_pairs;
  if (units == 0 || n_q == 0) return MLA_OK;
  CUtensorMap tq, tk, tpe, tv;
  // kv_rows may be 0 (every sequence empty); the maps still need one row
  const uint64_t rows = kv_rows > 0 ? (uint64_t)kv_rows : 1;
  const void* k_base = kv_rows > 0 ? k_nope : q;
  const void* v_base = kv_rows > 0 ? v : q;
  const void* pe_base = kv_rows > 0 ? pe : q;
  {
    // q as [n_q][H][192]: a box is 64 columns of one head for 128 query rows
    const uint64_t d[3] = {192, (uint64_t)H, (uint64_t)n_q}, st[2] = {384, (uint64_t)q_row_stride * 2};
    const uint32_t b[3] = {64, 1, (uint32_t)kFaTile};
    if (!make_map(&tq, q, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    // K_nope and V as [H][rows][128]: a box is 64 columns of 128 keys of one head
    const uint64_t d[3] = {128, rows, (uint64_t)H}, st[2] = {256, rows * 256};
    const uint32_t b[3] = {64, (uint32_t)kFaTile, 1};
    if (!make_map(&tk, k_base, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
    if (!make_map(&tv, v_base, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t d[2] = {64, rows}, st[1] = {128};
    const uint32_t b[2] = {64, (uint32_t)kFaTile};
    if (!make_map(&tpe, pe_base, 2, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B)) return MLA_ERR_CUDA;
  }
  FaParams p;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.heads = H;
  p.q_pairs = (int)q_pairs;
  p.n_units = units;
  p.n_q = n_q;
  p.kv_rows = kv_rows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  constexpr size_t smem = fa_smem_bytes();
  if (!set_smem(fmha_kernel, smem)) return MLA_ERR_CUDA;
  const int64_t grid = units < sms ? units : sms;
  return launch(true, fmha_kernel, dim3((unsigned)grid), dim3(kFaThreads), smem, stream, tq, tk, tpe, tv, p);
}

}  // namespace sm100
}  // namespace mla
