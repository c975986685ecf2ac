// mla_lib.cu -- the C ABI declared in include/mla.h: argument checks, kernel
// choice, workspace layout and launches.  Every arithmetic step runs in the
// kernels included below; this file only marshals.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "mla.h"
#ifdef MLA_FAULT_INJECT
#include "mla_fault_inject.h"
#endif
#include "common.cuh"
#include "simt.cuh"
#include "append.cuh"
#include "gather.cuh"
#include "sm100.cuh"

namespace {

using mla_bf16 = __nv_bfloat16;

struct Geo {
  int H, C, Dn, R, Dv;
  bool bf16;
  float scale;
  int family;   // 1 tensor-core kernels, 0 CUDA-core kernels, -1 unsupported
};

int pick_family(const mla_dims_t* d) {
  if (!d) return -1;
  if (d->num_heads <= 0 || d->kv_lora_rank <= 0 || d->qk_nope_head_dim <= 0 || d->qk_rope_head_dim < 0 ||
      d->v_head_dim <= 0)
    return -1;
  if (d->dtype != MLA_DTYPE_BF16 && d->dtype != MLA_DTYPE_F32) return -1;
  if (d->dtype == MLA_DTYPE_BF16 && mla::sm100::supports(d->num_heads, d->kv_lora_rank, d->qk_nope_head_dim,
                                                          d->qk_rope_head_dim, d->v_head_dim))
    return 1;
  if (d->kv_lora_rank > mla::simt::kMaxC || d->qk_rope_head_dim > mla::simt::kMaxR ||
      d->qk_nope_head_dim > mla::simt::kMaxD || d->v_head_dim > mla::simt::kMaxD || d->num_heads > 1024)
    return -1;
  return 0;
}

bool geo_of(const mla_dims_t* d, Geo* g) {
  g->family = pick_family(d);
  if (g->family < 0) return false;
  if (!(d->softmax_scale >= 0.f && d->softmax_scale < INFINITY)) return false;
  g->H = d->num_heads; g->C = d->kv_lora_rank; g->Dn = d->qk_nope_head_dim;
  g->R = d->qk_rope_head_dim; g->Dv = d->v_head_dim;
  g->bf16 = d->dtype == MLA_DTYPE_BF16;
  g->scale = d->softmax_scale;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status_t launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ---- split-t planning (CUDA-core kernels) ----------------------------------
int simt_auto_splits(int64_t n_q_rows, int H, int64_t max_seqlen_k) {
  const int64_t blocks = n_q_rows * H;
  const int64_t want = 4LL * device_sm_count();
  int splits = 1;
  while (splits < 64 && blocks * splits < want && max_seqlen_k / (splits * 2) >= 1024) splits *= 2;
  return splits;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Control words of mla_attn_decode_fused at the start of its workspace.
constexpr size_t kFusedCtrlBytes = 256;

size_t simt_workspace(const Geo& g, int64_t n_q_rows, int splits) {
  if (splits <= 1) return 0;
  return align256((size_t)splits * n_q_rows * g.H * g.C * sizeof(float)) +
         align256((size_t)splits * n_q_rows * g.H * 2 * sizeof(float));
}

template <typename T>
mla_status_t simt_attention(const Geo& g, const void* q_abs, const void* q, int64_t q_row_stride,
                            const void* kv, const void* pe, int64_t kv_rows, const int32_t* cu_q, const int32_t* cu_k,
                            int batch,
                            int64_t n_rows, int splits, void* o_lat, void* ws, cudaStream_t stream,
                            const mla::sm100::PagedKv& paged = mla::sm100::PagedKv{}) {
  float* part_o = nullptr;
  float* part_ml = nullptr;
  if (splits > 1) {
    part_o = static_cast<float*>(ws);
    part_ml = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                       align256((size_t)splits * n_rows * g.H * g.C * sizeof(float)));
  }
  dim3 grid((unsigned)n_rows, g.H, splits);
  const size_t smem = mla::simt::attn_smem_bytes(g.C, g.R);
  mla::simt::attn_kernel<T><<<grid, mla::simt::kThreads, smem, stream>>>(
      static_cast<const T*>(q_abs), static_cast<const T*>(q), q_row_stride, static_cast<const T*>(kv),
      static_cast<const T*>(pe), kv_rows, cu_q, cu_k, batch, paged.seqlens, paged.table, paged.stride, paged.page,
      n_rows, g.H, g.C, g.R, g.Dn, g.scale, splits, static_cast<T*>(o_lat), part_o, part_ml);
  if (splits > 1) {
    mla::simt::combine_kernel<T><<<dim3((unsigned)n_rows, g.H), mla::simt::kThreads, 0, stream>>>(
        part_o, part_ml, splits, n_rows, g.H, g.C, static_cast<T*>(o_lat));
  }
  return launch_status();
}

int resolve_splits(const Geo& g, int32_t batch, int64_t n_q_rows, int64_t max_seqlen_k, int32_t num_splits,
                   bool decode) {
  if (!decode) return g.family == 1 ? mla::sm100::prefill_splits() : 1;
  if (num_splits > 0) return num_splits;
  if (g.family == 1) return mla::sm100::auto_decode_splits(batch, g.H, max_seqlen_k, device_sm_count());
  return simt_auto_splits(n_q_rows, g.H, max_seqlen_k);
}

size_t workspace_bytes_for(const Geo& g, int32_t batch, int64_t n_q_rows, int64_t max_seqlen_k, int splits,
                           bool decode) {
  if (g.family == 1) return mla::sm100::workspace_bytes(g.H, n_q_rows, splits);
  return simt_workspace(g, n_q_rows, splits);
}

// Scratch for mla_attn_decode_static_scratch: one array per device that loads
// the library, for callers that cannot allocate.  Host code only ever uses
// the device address looked up below, never this symbol directly.
static __device__ __align__(256) unsigned char g_static_scratch[MLA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once per device).
void* static_scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

// Sparse decode workspace: the gathered latent and rotary rows (one page of `page` rows per
// sequence), the per-sequence key counts and block table, then the paged attention's workspace.
struct SparseLayout {
  int64_t page;
  size_t off_pe, off_lens, off_table, off_attn, total;
};

bool sparse_layout(const Geo& g, int32_t batch, int32_t max_topk, int32_t num_splits, SparseLayout* s) {
  const size_t esz = g.bf16 ? 2 : 4;
  if ((g.C * esz) % 16 != 0 || (g.R * esz) % 16 != 0 || g.C * esz > 2 * 32 * 16 || g.R * esz > 32 * 16)
    return false;
  s->page = g.family == 1 ? ((int64_t)max_topk + 127) / 128 * 128 : (max_topk > 0 ? max_topk : 1);
  if (s->page <= 0) s->page = 128;
  const size_t rows = (size_t)batch * (size_t)s->page;
  s->off_pe = align256(rows * g.C * esz);
  s->off_lens = s->off_pe + align256(rows * g.R * esz);
  s->off_table = s->off_lens + align256((size_t)batch * 4);
  s->off_attn = s->off_table + align256((size_t)batch * 4);
  const int splits = resolve_splits(g, batch, batch, max_topk, num_splits, true);
  s->total = s->off_attn + workspace_bytes_for(g, batch, batch, max_topk, splits, true);
  return true;
}

}  // namespace

extern "C" {

int32_t mla_api_version(void) { return MLA_API_VERSION; }

int32_t mla_kernel_family(const mla_dims_t* dims) { return pick_family(dims); }

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported head geometry or dtype";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

mla_status_t mla_absorb_q(const mla_dims_t* dims, const void* q, int64_t q_row_stride, const void* wkv_b,
                          void* q_abs, int64_t n_rows, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (n_rows < 0 || q_row_stride < (int64_t)g.H * (g.Dn + g.R)) return MLA_ERR_INVALID_ARG;
  if (n_rows == 0) return MLA_OK;
  if (!q || !wkv_b || !q_abs || !aligned16(q) || !aligned16(wkv_b) || !aligned16(q_abs)) return MLA_ERR_INVALID_ARG;
  if (g.family == 1) {
    if ((q_row_stride * 2) % 16 != 0) return MLA_ERR_INVALID_ARG;
    return mla::sm100::absorb_q(q, q_row_stride, wkv_b, q_abs, n_rows, g.H, stream);
  }
  dim3 grid((unsigned)((n_rows + mla::simt::kRowsPerBlock - 1) / mla::simt::kRowsPerBlock), g.H);
  if (g.bf16)
    mla::simt::absorb_q_kernel<mla_bf16><<<grid, mla::simt::kThreads, 0, stream>>>(
        static_cast<const mla_bf16*>(q), q_row_stride, static_cast<const mla_bf16*>(wkv_b),
        static_cast<mla_bf16*>(q_abs), n_rows, g.H, g.C, g.Dn, g.R, g.Dv);
  else
    mla::simt::absorb_q_kernel<float><<<grid, mla::simt::kThreads, 0, stream>>>(
        static_cast<const float*>(q), q_row_stride, static_cast<const float*>(wkv_b), static_cast<float*>(q_abs),
        n_rows, g.H, g.C, g.Dn, g.R, g.Dv);
  return launch_status();
}

mla_status_t mla_out_proj(const mla_dims_t* dims, const void* o_lat, const void* wkv_b, void* out, int64_t n_rows,
                          cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (n_rows < 0) return MLA_ERR_INVALID_ARG;
  if (n_rows == 0) return MLA_OK;
  if (!o_lat || !wkv_b || !out || !aligned16(o_lat) || !aligned16(wkv_b) || !aligned16(out))
    return MLA_ERR_INVALID_ARG;
  if (g.family == 1) return mla::sm100::out_proj(o_lat, wkv_b, out, n_rows, g.H, stream);
  dim3 grid((unsigned)((n_rows + mla::simt::kRowsPerBlock - 1) / mla::simt::kRowsPerBlock), g.H);
  size_t smem = (size_t)mla::simt::kRowsPerBlock * g.C * sizeof(float);
  if (g.bf16)
    mla::simt::out_proj_kernel<mla_bf16><<<grid, mla::simt::kThreads, smem, stream>>>(
        static_cast<const mla_bf16*>(o_lat), static_cast<const mla_bf16*>(wkv_b), static_cast<mla_bf16*>(out),
        n_rows, g.H, g.C, g.Dn, g.Dv);
  else
    mla::simt::out_proj_kernel<float><<<grid, mla::simt::kThreads, smem, stream>>>(
        static_cast<const float*>(o_lat), static_cast<const float*>(wkv_b), static_cast<float*>(out), n_rows, g.H,
        g.C, g.Dn, g.Dv);
  return launch_status();
}

size_t mla_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t n_q_rows, int64_t max_seqlen_k,
                          int32_t num_splits) {
  Geo g;
  if (!dims || !geo_of(dims, &g) || batch < 0 || n_q_rows < 0 || max_seqlen_k < 0 || num_splits < 0) return 0;
  // A decode call has exactly one query row per sequence.
  const bool decode = n_q_rows == batch;
  const int splits = resolve_splits(g, batch, n_q_rows, max_seqlen_k, num_splits, decode);
  size_t a = workspace_bytes_for(g, batch, n_q_rows, max_seqlen_k, splits, decode);
  if (decode) {
    // the same sizes may also be served as a chunked prefill
    size_t b = workspace_bytes_for(g, batch, n_q_rows, max_seqlen_k,
                                   resolve_splits(g, batch, n_q_rows, max_seqlen_k, 0, false), false);
    a = std::max(a, b);
  }
  return a;
}

int32_t mla_decode_num_splits(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k, int32_t num_splits) {
  Geo g;
  if (!dims || !geo_of(dims, &g) || batch < 0 || max_seqlen_k < 0 || num_splits < 0) return 0;
  return resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
}

mla_status_t mla_attn_decode(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                             const void* kv_cache, const void* pe_cache, int64_t kv_rows,
                             const int32_t* cu_seqlens_k, int32_t batch,
                             int64_t max_seqlen_k, void* o_lat, void* workspace, size_t workspace_bytes,
                             int32_t num_splits, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_seqlen_k < 0 || kv_rows < 0 || num_splits < 0 || num_splits > 256 ||
      q_row_stride < (int64_t)g.H * (g.Dn + g.R))
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q_abs || !q || !cu_seqlens_k || !o_lat || !aligned16(q_abs) || !aligned16(q) || !aligned16(o_lat))
    return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  const size_t need = workspace_bytes_for(g, batch, batch, max_seqlen_k, splits, true);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return MLA_ERR_WORKSPACE;
  if (g.family == 1) {
    if ((q_row_stride * 2) % 16 != 0) return MLA_ERR_INVALID_ARG;
    return mla::sm100::attention(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, nullptr, cu_seqlens_k, batch,
                                 batch, g.H, splits, g.scale, o_lat, workspace, stream);
  }
  if (g.bf16)
    return simt_attention<mla_bf16>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, nullptr, cu_seqlens_k,
                                    batch, batch, splits, o_lat, workspace, stream);
  return simt_attention<float>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, nullptr, cu_seqlens_k, batch,
                               batch, splits, o_lat, workspace, stream);
}

mla_status_t mla_attn_decode_static_scratch(const mla_dims_t* dims, const void* q_abs, const void* q,
                                            int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                            int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch,
                                            int64_t max_seqlen_k, void* o_lat, int32_t num_splits,
                                            cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_seqlen_k < 0 || num_splits < 0 || num_splits > 256) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  const size_t need = workspace_bytes_for(g, batch, batch, max_seqlen_k, splits, true);
  if (need > (size_t)MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    ws = static_scratch_for_current_device();
    if (!ws) return MLA_ERR_CUDA;
  }
  return mla_attn_decode(dims, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_k, batch,
                         max_seqlen_k, o_lat, ws, need > 0 ? (size_t)MLA_STATIC_SCRATCH_BYTES : 0, num_splits,
                         stream);
}

size_t mla_partials_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                   int32_t num_splits) {
  Geo g;
  if (!dims || !geo_of(dims, &g) || g.family != 1 || batch < 0 || max_seqlen_k < 0 || num_splits < 0 ||
      num_splits > 256)
    return 0;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  return mla::sm100::workspace_bytes(g.H, batch, splits, /*partials=*/true);
}

// Shared checks of the two merge calls: tensor-core dims, 1 <= num_splits <= 256, pointers.
static mla_status_t check_merge_args(const mla_dims_t* dims, const void* part_o, const void* part_ml,
                                     int32_t num_splits, int64_t n_q_rows, Geo* g) {
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, g)) return MLA_ERR_UNSUPPORTED;
  if (g->family != 1) return MLA_ERR_UNSUPPORTED;
  if (num_splits < 1 || num_splits > 256 || n_q_rows < 0 || n_q_rows >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  if (n_q_rows > 0 && (!part_o || !part_ml || !aligned16(part_o) || !aligned16(part_ml)))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

mla_status_t mla_merge_partials(const mla_dims_t* dims, const void* part_o, const void* part_ml,
                                int32_t num_splits, int64_t n_q_rows, void* o_lat, cudaStream_t stream) {
  Geo g;
  const mla_status_t st = check_merge_args(dims, part_o, part_ml, num_splits, n_q_rows, &g);
  if (st != MLA_OK) return st;
  if (n_q_rows == 0) return MLA_OK;
  if (!o_lat || !aligned16(o_lat)) return MLA_ERR_INVALID_ARG;
  return mla::sm100::merge_partials(part_o, part_ml, num_splits, n_q_rows, g.H, o_lat, stream);
}

mla_status_t mla_merge_partials_out(const mla_dims_t* dims, const void* part_o, const void* part_ml,
                                    int32_t num_splits, int64_t n_q_rows, const void* wkv_b, void* out,
                                    cudaStream_t stream) {
  Geo g;
  const mla_status_t st = check_merge_args(dims, part_o, part_ml, num_splits, n_q_rows, &g);
  if (st != MLA_OK) return st;
  if (n_q_rows == 0) return MLA_OK;
  if (!wkv_b || !out || !aligned16(wkv_b) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  return mla::sm100::merge_partials_out(part_o, part_ml, num_splits, n_q_rows, g.H, wkv_b, out, stream);
}

mla_status_t mla_attn_decode_partials(const mla_dims_t* dims, const void* q_abs, const void* q,
                                      int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                      int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch,
                                      int64_t max_seqlen_k, void* workspace, size_t workspace_bytes,
                                      int32_t num_splits, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (g.family != 1) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_seqlen_k < 0 || kv_rows < 0 || num_splits < 0 || num_splits > 256 ||
      q_row_stride < (int64_t)g.H * (g.Dn + g.R) || (q_row_stride * 2) % 16 != 0)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q_abs || !q || !cu_seqlens_k || !aligned16(q_abs) || !aligned16(q)) return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  const size_t need = mla::sm100::workspace_bytes(g.H, batch, splits, /*partials=*/true);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return MLA_ERR_WORKSPACE;
  return mla::sm100::attention(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, nullptr, cu_seqlens_k, batch,
                               batch, g.H, splits, g.scale, nullptr, workspace, stream, /*merge=*/false,
                               mla::sm100::PagedKv{}, /*partials=*/true);
}

size_t mla_decode_out_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                     int32_t num_splits) {
  Geo g;
  if (!dims || !geo_of(dims, &g) || batch < 0 || max_seqlen_k < 0 || num_splits < 0 || num_splits > 256) return 0;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  const size_t o_lat_bytes = align256((size_t)batch * g.H * g.C * (g.bf16 ? 2 : 4));
  return o_lat_bytes + workspace_bytes_for(g, batch, batch, max_seqlen_k, splits, true);
}

mla_status_t mla_attn_decode_out(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                 const void* kv_cache, const void* pe_cache, int64_t kv_rows,
                                 const int32_t* cu_seqlens_k, int32_t batch, int64_t max_seqlen_k,
                                 const void* wkv_b, void* out, void* workspace, size_t workspace_bytes,
                                 int32_t num_splits, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_seqlen_k < 0 || kv_rows < 0 || num_splits < 0 || num_splits > 256 ||
      q_row_stride < (int64_t)g.H * (g.Dn + g.R))
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q_abs || !q || !cu_seqlens_k || !wkv_b || !out || !aligned16(q_abs) || !aligned16(q) ||
      !aligned16(wkv_b) || !aligned16(out))
    return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_decode_out_workspace_size(dims, batch, max_seqlen_k, num_splits);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return MLA_ERR_WORKSPACE;
  // o_lat first, then the attention call's own workspace
  const size_t o_lat_bytes = align256((size_t)batch * g.H * g.C * (g.bf16 ? 2 : 4));
  void* o_lat = workspace;
  void* ws = static_cast<char*>(workspace) + o_lat_bytes;
  const size_t ws_bytes = workspace_bytes - o_lat_bytes;
  if (g.family == 1) {
    if ((q_row_stride * 2) % 16 != 0) return MLA_ERR_INVALID_ARG;
    const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
    // with splits the merge runs inside the projection kernel and o_lat is never written
    mla_status_t st = mla::sm100::attention(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, nullptr,
                                            cu_seqlens_k, batch, batch, g.H, splits, g.scale, o_lat, ws, stream,
                                            /*merge=*/splits <= 1);
    if (st != MLA_OK) return st;
    if (splits > 1) return mla::sm100::merge_out_proj(ws, splits, batch, g.H, wkv_b, out, stream);
    return mla::sm100::out_proj(o_lat, wkv_b, out, batch, g.H, stream);
  }
  mla_status_t st = mla_attn_decode(dims, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_k, batch,
                                    max_seqlen_k, o_lat, ws, ws_bytes, num_splits, stream);
  if (st != MLA_OK) return st;
  return mla_out_proj(dims, o_lat, wkv_b, out, batch, stream);
}

size_t mla_decode_fused_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                       int32_t num_splits) {
  Geo g;
  if (!dims || !geo_of(dims, &g) || batch < 0 || max_seqlen_k < 0 || num_splits < 0 || num_splits > 256) return 0;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  size_t rest = mla_decode_out_workspace_size(dims, batch, max_seqlen_k, num_splits);
  if (g.family == 1) rest = std::max(rest, mla::sm100::workspace_bytes(g.H, batch, splits, /*partials=*/true));
  return kFusedCtrlBytes + rest;
}

mla_status_t mla_attn_decode_fused(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                   const void* kv_cache, const void* pe_cache, int64_t kv_rows,
                                   const int32_t* cu_seqlens_k, int32_t batch, int64_t max_seqlen_k,
                                   const void* wkv_b, void* out, void* workspace, size_t workspace_bytes,
                                   int32_t num_splits, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_seqlen_k < 0 || kv_rows < 0 || num_splits < 0 || num_splits > 256 ||
      q_row_stride < (int64_t)g.H * (g.Dn + g.R))
    return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const size_t need = mla_decode_fused_workspace_size(dims, batch, max_seqlen_k, num_splits);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return MLA_ERR_WORKSPACE;
  if (!q_abs || !q || !cu_seqlens_k || !wkv_b || !out || !aligned16(q_abs) || !aligned16(q) ||
      !aligned16(wkv_b) || !aligned16(out))
    return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  uint32_t* ctrl = static_cast<uint32_t*>(workspace);
  void* rest = static_cast<char*>(workspace) + kFusedCtrlBytes;
  const size_t rest_bytes = workspace_bytes - kFusedCtrlBytes;
  const int splits = resolve_splits(g, batch, batch, max_seqlen_k, num_splits, true);
  if (g.family == 1 && (q_row_stride * 2) % 16 == 0 && mla::sm100::fused_fits(batch, g.H, splits, device_sm_count()))
    return mla::sm100::decode_fused(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_k, batch, g.H,
                                    splits, g.scale, wkv_b, out, rest, ctrl, stream);
  // more units than can be resident at once, or a single split: the two-kernel path
  return mla_attn_decode_out(dims, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_k, batch,
                             max_seqlen_k, wkv_b, out, rest, rest_bytes, num_splits, stream);
}

mla_status_t mla_attn_prefill_chunk(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                                    int64_t n_q_rows, int64_t max_seqlen_q, int64_t max_seqlen_k,
                                    const void* kv_cache, const void* pe_cache, int64_t kv_rows, void* o_lat,
                                    void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || n_q_rows < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || kv_rows < 0 ||
      q_row_stride < (int64_t)g.H * (g.Dn + g.R))
    return MLA_ERR_INVALID_ARG;
  if (batch == 0 || n_q_rows == 0) return MLA_OK;
  if (!q_abs || !q || !cu_seqlens_q || !cu_seqlens_k || !o_lat || !aligned16(q_abs) || !aligned16(q) ||
      !aligned16(o_lat))
    return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  const int splits = resolve_splits(g, batch, n_q_rows, max_seqlen_k, 0, false);
  const size_t need = workspace_bytes_for(g, batch, n_q_rows, max_seqlen_k, splits, false);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return MLA_ERR_WORKSPACE;
  if (g.family == 1) {
    if ((q_row_stride * 2) % 16 != 0) return MLA_ERR_INVALID_ARG;
    return mla::sm100::attention(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q, cu_seqlens_k,
                                 batch, n_q_rows, g.H, splits, g.scale, o_lat, workspace, stream);
  }
  if (g.bf16)
    return simt_attention<mla_bf16>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q,
                                    cu_seqlens_k, batch, n_q_rows, splits, o_lat, workspace, stream);
  return simt_attention<float>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q, cu_seqlens_k,
                               batch, n_q_rows, splits, o_lat, workspace, stream);
}

mla_status_t mla_attn_prefill_expanded(const mla_dims_t* dims, const void* q, int64_t q_row_stride,
                                       const void* k_nope, const void* v, const void* pe_cache, int64_t kv_rows,
                                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                                       int64_t n_q_rows, int64_t max_seqlen_q, void* out, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (g.family != 1) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || n_q_rows < 0 || max_seqlen_q < 0 || kv_rows < 0 || q_row_stride < (int64_t)g.H * (g.Dn + g.R) ||
      (q_row_stride * 2) % 16 != 0)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0 || n_q_rows == 0) return MLA_OK;
  if (!q || !cu_seqlens_q || !cu_seqlens_k || !out || !aligned16(q) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!k_nope || !v || !pe_cache || !aligned16(k_nope) || !aligned16(v) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  return mla::sm100::attention_expanded(q, q_row_stride, k_nope, v, pe_cache, kv_rows, cu_seqlens_q, cu_seqlens_k,
                                        batch, n_q_rows, max_seqlen_q, g.H, g.scale, out, device_sm_count(), stream);
}

// mla_attn_paged; early_cache = false when the kernel just before the attention writes the cache
// (the sparse path's row gather), so the attention must not read it before waiting for that kernel.
static mla_status_t attn_paged_impl(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                    const int32_t* cu_seqlens_q, int64_t n_q_rows, const int32_t* seqlens_k,
                                    int32_t batch, int64_t max_seqlen_k, const void* kv_cache, const void* pe_cache,
                                    int64_t num_pages, int32_t page_size, const int32_t* block_table,
                                    int64_t max_pages_per_seq, void* o_lat, void* workspace, size_t workspace_bytes,
                                    int32_t num_splits, cudaStream_t stream, bool early_cache) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  const bool decode = cu_seqlens_q == nullptr;
  if (batch < 0 || n_q_rows < 0 || max_seqlen_k < 0 || num_pages < 0 || page_size <= 0 || max_pages_per_seq < 0 ||
      num_splits < 0 || num_splits > 256 || q_row_stride < (int64_t)g.H * (g.Dn + g.R) ||
      (decode && n_q_rows != batch) || (!decode && num_splits > 1))
    return MLA_ERR_INVALID_ARG;
  if (num_pages > (int64_t{1} << 40) / page_size) return MLA_ERR_INVALID_ARG;
  const int64_t kv_rows = num_pages * page_size;
  if (g.family == 1 && page_size % 64 != 0) return MLA_ERR_UNSUPPORTED;
  if (batch == 0 || n_q_rows == 0) return MLA_OK;
  if (!q_abs || !q || !seqlens_k || !block_table || !o_lat || !aligned16(q_abs) || !aligned16(q) ||
      !aligned16(o_lat))
    return MLA_ERR_INVALID_ARG;
  if (kv_rows > 0 && (!kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  const int splits = resolve_splits(g, batch, n_q_rows, max_seqlen_k, num_splits, decode);
  const size_t need = workspace_bytes_for(g, batch, n_q_rows, max_seqlen_k, splits, decode);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return MLA_ERR_WORKSPACE;
  mla::sm100::PagedKv paged;
  paged.seqlens = seqlens_k;
  paged.table = block_table;
  paged.stride = max_pages_per_seq;
  paged.page = page_size;
  if (g.family == 1) {
    if ((q_row_stride * 2) % 16 != 0) return MLA_ERR_INVALID_ARG;
    return mla::sm100::attention(q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q, nullptr, batch,
                                 n_q_rows, g.H, splits, g.scale, o_lat, workspace, stream, true, paged,
                                 /*partials=*/false, early_cache);
  }
  if (g.bf16)
    return simt_attention<mla_bf16>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q, nullptr,
                                    batch, n_q_rows, splits, o_lat, workspace, stream, paged);
  return simt_attention<float>(g, q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, cu_seqlens_q, nullptr, batch,
                               n_q_rows, splits, o_lat, workspace, stream, paged);
}

mla_status_t mla_attn_paged(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                            const int32_t* cu_seqlens_q, int64_t n_q_rows, const int32_t* seqlens_k, int32_t batch,
                            int64_t max_seqlen_k, const void* kv_cache, const void* pe_cache, int64_t num_pages,
                            int32_t page_size, const int32_t* block_table, int64_t max_pages_per_seq, void* o_lat,
                            void* workspace, size_t workspace_bytes, int32_t num_splits, cudaStream_t stream) {
  return attn_paged_impl(dims, q_abs, q, q_row_stride, cu_seqlens_q, n_q_rows, seqlens_k, batch, max_seqlen_k,
                         kv_cache, pe_cache, num_pages, page_size, block_table, max_pages_per_seq, o_lat, workspace,
                         workspace_bytes, num_splits, stream, /*early_cache=*/true);
}

size_t mla_sparse_workspace_size(const mla_dims_t* dims, int32_t batch, int32_t max_topk, int32_t num_splits) {
  Geo g;
  SparseLayout sl;
  if (!dims || !geo_of(dims, &g) || batch < 0 || max_topk < 0 || num_splits < 0 || num_splits > 256) return 0;
  if (!sparse_layout(g, batch, max_topk, num_splits, &sl)) return 0;
  return sl.total;
}

mla_status_t mla_attn_sparse_decode(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                    const void* kv_cache, const void* pe_cache, int64_t kv_rows,
                                    const int32_t* indices, int64_t index_stride, const int32_t* counts,
                                    int32_t batch, int32_t max_topk, void* o_lat, void* workspace,
                                    size_t workspace_bytes, int32_t num_splits, cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || max_topk < 0 || kv_rows < 0 || num_splits < 0 || num_splits > 256 ||
      index_stride < max_topk || q_row_stride < (int64_t)g.H * (g.Dn + g.R))
    return MLA_ERR_INVALID_ARG;
  SparseLayout sl;
  if (!sparse_layout(g, batch, max_topk, num_splits, &sl)) return MLA_ERR_UNSUPPORTED;
  if (batch == 0) return MLA_OK;
  if ((int64_t)batch * sl.page >= (1LL << 31) || batch > 65535) return MLA_ERR_INVALID_ARG;
  if (!q_abs || !q || !counts || !o_lat || !aligned16(q_abs) || !aligned16(q) || !aligned16(o_lat))
    return MLA_ERR_INVALID_ARG;
  if (max_topk > 0 && (!indices || !kv_cache || !pe_cache || !aligned16(kv_cache) || !aligned16(pe_cache)))
    return MLA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < sl.total || !aligned16(workspace)) return MLA_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  void* kv_sel = ws;
  void* pe_sel = ws + sl.off_pe;
  int32_t* lens = reinterpret_cast<int32_t*>(ws + sl.off_lens);
  int32_t* table = reinterpret_cast<int32_t*>(ws + sl.off_table);
  const size_t esz = g.bf16 ? 2 : 4;
  const int kv_vec = (int)(g.C * esz / 16), pe_vec = (int)(g.R * esz / 16);
  const int64_t per_block = mla::gather::kWarps;
  int64_t bx = max_topk > 0 ? (max_topk + per_block - 1) / per_block : 1;
  if (bx > 64) bx = 64;
  mla::gather::select_rows_kernel<<<dim3((unsigned)bx, (unsigned)batch), mla::gather::kWarps * 32, 0, stream>>>(
      static_cast<const uint4*>(kv_cache), static_cast<const uint4*>(pe_cache), kv_rows, indices, index_stride,
      counts, max_topk, sl.page, kv_vec, pe_vec, static_cast<uint4*>(kv_sel), static_cast<uint4*>(pe_sel), lens,
      table);
  if (launch_status() != MLA_OK) return MLA_ERR_CUDA;
  // the paged attention over one page per sequence: block table entry b = page b
  return attn_paged_impl(dims, q_abs, q, q_row_stride, nullptr, batch, lens, batch, max_topk, kv_sel, pe_sel, batch,
                         (int32_t)sl.page, table, 1, o_lat, ws + sl.off_attn, sl.total - sl.off_attn, num_splits,
                         stream, /*early_cache=*/false);
}

mla_status_t mla_expand_kv(const mla_dims_t* dims, const void* kv_c, const void* gamma, float eps,
                           const void* wkv_b, int64_t batch, int64_t seq_len, void* k_nope, void* v,
                           cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  if (batch < 0 || seq_len < 0 || !(eps >= 0.f && eps < INFINITY)) return MLA_ERR_INVALID_ARG;
  if (batch > 0 && seq_len > ((int64_t)1 << 40) / batch) return MLA_ERR_INVALID_ARG;
  const int64_t n_tokens = batch * seq_len;
  if (n_tokens == 0) return MLA_OK;
  if (!kv_c || !wkv_b || !k_nope || !v || !aligned16(kv_c) || !aligned16(wkv_b) || !aligned16(k_nope) ||
      !aligned16(v) || (gamma && !aligned16(gamma)))
    return MLA_ERR_INVALID_ARG;
  if (g.family == 1)
    return mla::sm100::expand_kv(kv_c, gamma, eps, wkv_b, batch, seq_len, g.H, k_nope, v, device_sm_count(),
                                 stream);
  if (n_tokens >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  const dim3 grid((unsigned)n_tokens, g.H);
  const size_t smem = (size_t)(g.C + 32) * sizeof(float);
  if (g.bf16)
    mla::simt::expand_kernel<mla_bf16><<<grid, mla::simt::kThreads, smem, stream>>>(
        static_cast<const mla_bf16*>(kv_c), static_cast<const mla_bf16*>(gamma), eps,
        static_cast<const mla_bf16*>(wkv_b), seq_len, g.H, g.C, g.Dn, g.Dv, static_cast<mla_bf16*>(k_nope),
        static_cast<mla_bf16*>(v));
  else
    mla::simt::expand_kernel<float><<<grid, mla::simt::kThreads, smem, stream>>>(
        static_cast<const float*>(kv_c), static_cast<const float*>(gamma), eps, static_cast<const float*>(wkv_b),
        seq_len, g.H, g.C, g.Dn, g.Dv, static_cast<float*>(k_nope), static_cast<float*>(v));
  return launch_status();
}

mla_status_t mla_append_latent(const mla_dims_t* dims, const void* kv_new, const void* k_pe_new, const void* gamma,
                               float eps, float rope_base, const int32_t* positions, const int64_t* slots,
                               int64_t n_tokens, void* kv_cache, void* pe_cache, int64_t cache_rows,
                               cudaStream_t stream) {
  Geo g;
  if (!dims) return MLA_ERR_INVALID_ARG;
  if (!geo_of(dims, &g)) return MLA_ERR_UNSUPPORTED;
  const int vec = g.bf16 ? 8 : 4;
  if (g.C % vec != 0 || g.C > mla::append::kMaxC || g.R % 2 != 0 || g.R > 64 * mla::append::kMaxPairsPerLane)
    return MLA_ERR_UNSUPPORTED;
  if (n_tokens < 0 || cache_rows < 0 || !(eps >= 0.f && eps < INFINITY) || !(rope_base > 0.f && rope_base < INFINITY))
    return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!kv_new || !k_pe_new || !positions || !slots || !kv_cache || !pe_cache || !aligned16(kv_new) ||
      !aligned16(kv_cache) || (gamma && !aligned16(gamma)))
    return MLA_ERR_INVALID_ARG;
  const int64_t per_block = (int64_t)mla::append::kWarpsPerBlock * mla::append::kTokensPerWarp;
  const int64_t nblocks = (n_tokens + per_block - 1) / per_block;
  if (nblocks >= (1LL << 31)) return MLA_ERR_INVALID_ARG;
  const unsigned blocks = (unsigned)nblocks;
  const double log2_base = std::log2((double)rope_base);
  const dim3 block(mla::append::kWarpsPerBlock * 32);
  auto go = [&](auto type_tag, auto per_lane) {
    using T = decltype(type_tag);
    constexpr int P = decltype(per_lane)::value;
    mla::append::append_kernel<T, P><<<blocks, block, 0, stream>>>(
        static_cast<const T*>(kv_new), static_cast<const T*>(k_pe_new), static_cast<const T*>(gamma), eps,
        log2_base, positions, slots, n_tokens, g.C, g.R, static_cast<T*>(kv_cache), static_cast<T*>(pe_cache),
        cache_rows);
  };
  // 16-byte vectors per lane: bf16 rows hold 8 elements per vector, fp32 rows 4
  const int per_lane = (g.C / vec + 31) / 32;
  using I1 = std::integral_constant<int, 1>;
  using I2 = std::integral_constant<int, 2>;
  using I4 = std::integral_constant<int, 4>;
  using I8 = std::integral_constant<int, 8>;
  if (g.bf16) {
    if (per_lane <= 1) go(mla_bf16{}, I1{});
    else if (per_lane <= 2) go(mla_bf16{}, I2{});
    else go(mla_bf16{}, I4{});
  } else {
    if (per_lane <= 1) go(0.f, I1{});
    else if (per_lane <= 2) go(0.f, I2{});
    else if (per_lane <= 4) go(0.f, I4{});
    else go(0.f, I8{});
  }
  return launch_status();
}

#ifdef MLA_FAULT_INJECT
// Fault-injection build only (tests of the bounded waits): set the plan word the kernels read.
mla_status_t mla_test_set_fault_plan(uint32_t plan) {
  return cudaMemcpyToSymbol(mla::g_mla_fault_plan, &plan, sizeof(plan)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
#endif

mla_status_t mla_device_status(cudaStream_t stream, uint32_t* code_out) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, mla::g_mla_error_word, sizeof(word)) != cudaSuccess) return MLA_ERR_CUDA;
  if (code_out) *code_out = word;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(mla::g_mla_error_word, &zero, sizeof(zero)) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_ERR_DEVICE_TIMEOUT;
  }
  return MLA_OK;
}

}  // extern "C"
