// simt.cuh -- CUDA-core kernels for any head geometry, fp32 or bf16 storage,
// fp32 arithmetic.  They serve the fp32 dtype (whose 1e-5 relative bound no
// bf16/TF32 tensor-core product meets) and bf16 shapes the tensor-core kernels
// are not built for.
//
// Operation: "Naive vs Absorb Attention Implementations in DeepSeek-V3",
// section "Absorb Path Execution" (absorbed query, two-term scores, latent
// value sum, output up-projection), with a softmax over the visible keys.
#pragma once

#include "common.cuh"

namespace mla {
namespace simt {

constexpr int kThreads = 128;
constexpr int kRowsPerBlock = 8;   // query rows sharing one weight read in the projections
constexpr int kMaxC = 1024, kMaxR = 128, kMaxD = 256;

// q_abs[n,h,c] = sum_{d<Dn} q[n,h,d] * W[h,d,c].  grid (ceil(n/8), H), 128 threads.
template <typename T>
__global__ void __launch_bounds__(kThreads) absorb_q_kernel(
    const T* __restrict__ q, int64_t q_row_stride, const T* __restrict__ wkv_b, T* __restrict__ q_abs,
    int64_t n_rows, int H, int C, int Dn, int R, int Dv) {
  __shared__ float qn[kRowsPerBlock][kMaxD];
  const int h = blockIdx.y;
  const int64_t n0 = (int64_t)blockIdx.x * kRowsPerBlock;
  const int rows = (int)min64(kRowsPerBlock, n_rows - n0);
  for (int i = threadIdx.x; i < kRowsPerBlock * Dn; i += kThreads) {
    int r = i / Dn, d = i % Dn;
    qn[r][d] = r < rows ? Elem<T>::load(q + (n0 + r) * q_row_stride + (int64_t)h * (Dn + R) + d) : 0.f;
  }
  __syncthreads();
  const T* w = wkv_b + (int64_t)h * (Dn + Dv) * C;
  for (int c = threadIdx.x; c < C; c += kThreads) {
    float acc[kRowsPerBlock];
#pragma unroll
    for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = 0.f;
    for (int d = 0; d < Dn; ++d) {
      float wv = Elem<T>::load(w + (int64_t)d * C + c);
#pragma unroll
      for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = fmaf(qn[r][d], wv, acc[r]);
    }
    for (int r = 0; r < rows; ++r) Elem<T>::store(q_abs + ((n0 + r) * H + h) * (int64_t)C + c, acc[r]);
  }
}

// out[n,h,d] = sum_c o_lat[n,h,c] * W[h,Dn+d,c].  grid (ceil(n/8), H), 128 threads.
template <typename T>
__global__ void __launch_bounds__(kThreads) out_proj_kernel(
    const T* __restrict__ o_lat, const T* __restrict__ wkv_b, T* __restrict__ out, int64_t n_rows, int H,
    int C, int Dn, int Dv) {
  extern __shared__ float o_s[];   // [kRowsPerBlock][C]
  const int h = blockIdx.y;
  const int64_t n0 = (int64_t)blockIdx.x * kRowsPerBlock;
  const int rows = (int)min64(kRowsPerBlock, n_rows - n0);
  for (int i = threadIdx.x; i < kRowsPerBlock * C; i += kThreads) {
    int r = i / C, c = i % C;
    o_s[i] = r < rows ? Elem<T>::load(o_lat + ((n0 + r) * H + h) * (int64_t)C + c) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* w = wkv_b + ((int64_t)h * (Dn + Dv) + Dn) * C;
  for (int d = warp; d < Dv; d += kThreads / 32) {
    float acc[kRowsPerBlock];
#pragma unroll
    for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = 0.f;
    for (int c = lane; c < C; c += 32) {
      float wv = Elem<T>::load(w + (int64_t)d * C + c);
#pragma unroll
      for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = fmaf(o_s[r * C + c], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = warp_sum(acc[r]);
    if (lane == 0)
      for (int r = 0; r < rows; ++r) Elem<T>::store(out + ((n0 + r) * H + h) * (int64_t)Dv + d, acc[r]);
  }
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  v = warp_max(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}
__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < kThreads / 32; ++i) r += red[i];
  return r;
}

// Shared memory of attn_kernel in bytes: floats q_abs [C], q_pe [R], o [C], p [kThreads],
// reduction scratch [32], then the cache row of each key of a chunk (int64 [kThreads]).
__host__ __device__ constexpr size_t attn_floats(int C, int R) { return ((size_t)2 * C + R + kThreads + 32 + 1) & ~(size_t)1; }
__host__ __device__ constexpr size_t attn_smem_bytes(int C, int R) {
  return attn_floats(C, R) * sizeof(float) + kThreads * sizeof(int64_t);
}

// Attention for one (query row, head, split) per block, online softmax over
// 128-key chunks.  With num_splits == 1 the normalised result goes straight to
// o_lat; otherwise the unnormalised partial (o, running max m, running sum l)
// goes to the workspace for attn_combine_kernel.  Keys visible to query i of
// a chunk of s over a cache of t: j < t - s + i + 1.  The cache is packed
// (sequence b's keys in rows cu_k[b] ..) or, with a block table, paged: key j
// in row table[b][j / page] * page + j % page; a page outside the cache reads
// as zeros and raises kErrBadPage.
template <typename T>
__global__ void __launch_bounds__(kThreads) attn_kernel(
    const T* __restrict__ q_abs, const T* __restrict__ q, int64_t q_row_stride, const T* __restrict__ kv,
    const T* __restrict__ pe, int64_t kv_rows, const int* __restrict__ cu_q, const int* __restrict__ cu_k, int batch,
    const int* __restrict__ seqlens_k, const int* __restrict__ block_table, int64_t bt_stride, int page_size,
    int64_t n_rows, int H, int C, int R, int Dn, float scale, int num_splits, T* __restrict__ o_lat,
    float* __restrict__ part_o, float* __restrict__ part_ml) {
  extern __shared__ float sm[];
  float* qa = sm;            // [C]
  float* qp = qa + C;        // [R]
  float* o = qp + R;         // [C]
  float* p = o + C;          // [kThreads]
  float* red = p + kThreads; // [32]
  int64_t* krow = reinterpret_cast<int64_t*>(sm + attn_floats(C, R));   // [kThreads], -1 = zero row
  const int64_t n = blockIdx.x;
  const int h = blockIdx.y, split = blockIdx.z;
  const int b = cu_q ? find_sequence(cu_q, batch, n) : (int)n;
  int64_t k0, t;
  const int* bt = nullptr;
  if (block_table) {
    bt = block_table + (int64_t)b * bt_stride;
    k0 = 0;
    t = max64(0, min64((int64_t)__ldg(seqlens_k + b), bt_stride * page_size));
  } else {
    k0 = min64(max64(0, __ldg(cu_k + b)), kv_rows);
    t = max64(0, min64((int64_t)__ldg(cu_k + b + 1), kv_rows) - k0);
  }
  int64_t s = 1, i = 0;
  if (cu_q) {
    const int64_t q0 = __ldg(cu_q + b);
    s = max64(0, (int64_t)__ldg(cu_q + b + 1) - q0);
    i = n - q0;
  }
  const int64_t visible = min64(t, max64(0, t - s + i + 1));
  const int64_t per = (visible + num_splits - 1) / num_splits;
  const int64_t j_begin = min64(visible, (int64_t)split * per);
  const int64_t j_end = min64(visible, j_begin + per);

  for (int c = threadIdx.x; c < C; c += kThreads) {
    qa[c] = Elem<T>::load(q_abs + (n * H + h) * (int64_t)C + c);
    o[c] = 0.f;
  }
  for (int r = threadIdx.x; r < R; r += kThreads)
    qp[r] = Elem<T>::load(q + n * q_row_stride + (int64_t)h * (Dn + R) + Dn + r);
  __syncthreads();

  float m = -INFINITY, l = 0.f;
  for (int64_t j0 = j_begin; j0 < j_end; j0 += kThreads) {
    const int64_t j = j0 + threadIdx.x;
    float sc = -INFINITY;
    if (j < j_end) {
      int64_t row = k0 + j;
      if (bt) {
        const int e = __ldg(bt + j / page_size);
        row = (e < 0 || ((int64_t)e + 1) * page_size > kv_rows) ? -1 : (int64_t)e * page_size + j % page_size;
        if (row < 0) raise_error(kErrBadPage);
      }
      krow[threadIdx.x] = row;
      float acc = 0.f;
      if (row >= 0) {
        const T* kr = kv + row * (int64_t)C;
        const T* pr = pe + row * (int64_t)R;
        for (int c = 0; c < C; ++c) acc = fmaf(qa[c], Elem<T>::load(kr + c), acc);
        for (int r = 0; r < R; ++r) acc = fmaf(qp[r], Elem<T>::load(pr + r), acc);
      }
      sc = acc * scale;
    }
    const float cmax = block_reduce_max(sc, red);
    const float m_new = fmaxf(m, cmax);
    const float alpha = expf(m - m_new);   // m = -inf on the first chunk gives 0
    const float pj = (j < j_end) ? expf(sc - m_new) : 0.f;
    p[threadIdx.x] = pj;
    const float psum = block_reduce_sum(pj, red);   // also orders the p[] writes
    l = l * alpha + psum;
    m = m_new;
    const int cnt = (int)min64(kThreads, j_end - j0);
    for (int c = threadIdx.x; c < C; c += kThreads) {
      float acc = o[c] * alpha;
      for (int jj = 0; jj < cnt; ++jj)
        if (krow[jj] >= 0) acc = fmaf(p[jj], Elem<T>::load(kv + krow[jj] * (int64_t)C + c), acc);
      o[c] = acc;
    }
    __syncthreads();
  }

  if (num_splits == 1) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int c = threadIdx.x; c < C; c += kThreads) Elem<T>::store(o_lat + (n * H + h) * (int64_t)C + c, o[c] * inv);
  } else {
    const int64_t slot = ((int64_t)split * n_rows + n) * H + h;
    for (int c = threadIdx.x; c < C; c += kThreads) part_o[slot * C + c] = o[c];
    if (threadIdx.x == 0) {
      part_ml[slot * 2 + 0] = m;
      part_ml[slot * 2 + 1] = l;
    }
  }
}

// Merge split partials: o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s, M = max_s m_s.
// grid (n_rows, H), 128 threads.  A row with no key anywhere gets zeros.
template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_ml, int num_splits, int64_t n_rows,
    int H, int C, T* __restrict__ o_lat) {
  const int64_t n = blockIdx.x;
  const int h = blockIdx.y;
  float mx = -INFINITY;
  for (int s = 0; s < num_splits; ++s) mx = fmaxf(mx, part_ml[(((int64_t)s * n_rows + n) * H + h) * 2]);
  float L = 0.f;
  for (int s = 0; s < num_splits; ++s) {
    const int64_t slot = ((int64_t)s * n_rows + n) * H + h;
    const float ms = part_ml[slot * 2];
    if (ms != -INFINITY) L += expf(ms - mx) * part_ml[slot * 2 + 1];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int c = threadIdx.x; c < C; c += kThreads) {
    float acc = 0.f;
    for (int s = 0; s < num_splits; ++s) {
      const int64_t slot = ((int64_t)s * n_rows + n) * H + h;
      const float ms = part_ml[slot * 2];
      if (ms != -INFINITY) acc = fmaf(expf(ms - mx), part_o[slot * C + c], acc);
    }
    Elem<T>::store(o_lat + (n * H + h) * (int64_t)C + c, acc * inv);
  }
}

// Latent KV expansion for one (token, head) per block: x = kv_c[tok] / sqrt(mean(kv_c[tok]^2) + eps)
// * gamma, then the head's Dn key rows and Dv value rows of wkv_b against x.  Outputs
// [batch, H, seq_len, Dn] and [batch, H, seq_len, Dv]; grid (tokens, H), 128 threads,
// shared memory (C + 32) floats.
template <typename T>
__global__ void __launch_bounds__(kThreads) expand_kernel(
    const T* __restrict__ kv_c, const T* __restrict__ gamma, float eps, const T* __restrict__ wkv_b,
    int64_t seq_len, int H, int C, int Dn, int Dv, T* __restrict__ k_nope, T* __restrict__ v) {
  extern __shared__ float xs[];   // [C]
  float* red = xs + C;            // [32]
  const int64_t tok = blockIdx.x;
  const int h = blockIdx.y;
  float ss = 0.f;
  for (int c = threadIdx.x; c < C; c += kThreads) {
    const float x = Elem<T>::load(kv_c + tok * C + c);
    xs[c] = x;
    ss = fmaf(x, x, ss);
  }
  ss = block_reduce_sum(ss, red);
  const float r = rsqrtf(ss / (float)C + eps);
  for (int c = threadIdx.x; c < C; c += kThreads) xs[c] *= r * (gamma ? Elem<T>::load(gamma + c) : 1.f);
  __syncthreads();
  const int64_t b = tok / seq_len, s = tok % seq_len;
  const T* w = wkv_b + (int64_t)h * (Dn + Dv) * C;
  for (int d = threadIdx.x; d < Dn + Dv; d += kThreads) {
    float acc = 0.f;
    for (int c = 0; c < C; ++c) acc = fmaf(xs[c], Elem<T>::load(w + (int64_t)d * C + c), acc);
    if (d < Dn)
      Elem<T>::store(k_nope + ((b * H + h) * seq_len + s) * Dn + d, acc);
    else
      Elem<T>::store(v + ((b * H + h) * seq_len + s) * Dv + (d - Dn), acc);
  }
}

}  // namespace simt
}  // namespace mla
